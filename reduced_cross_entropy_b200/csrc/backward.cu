// backward.cu -- step 6 of the path: gradients of the reduced loss (RECE, equation 4,
// restricted to the positive and the kept negatives; selection held constant).
//
//   g_ij = (exp(l_ij - lse_i) - [j == z_i]) * dloss / N
//   (the sampled baselines reuse it: CE- with its sampled negatives in the slots, BCE+
//   with sigmoid(l_ij) in place of the softmax term; see sampled.cu)
//   dX_i = sum_j g_ij y_j          (one warp per row: every lane computes whole dot
//                                   products for its own slots, then the lanes sweep the
//                                   dimensions adding the slots in order)
//   dY_j = sum_i g_ij x_i          (no float atomics: the (item, row) pairs are put in
//                                   item order by a stable LSD radix sort of (item, pair
//                                   id), then one warp per item sums its pairs in row
//                                   order, fetching each pair's g by its id -- or, when
//                                   the g array is too large for L2, g rides along in
//                                   the sort; an item with a long run is summed by a
//                                   CTA, its warps' parts added in warp order)
// Pair e = i*(k+1) + s holds slot s of row i (s = 0: the positive, s >= 1: selected
// negative s-1); an empty slot carries the key C, which sorts after every item.  Every
// sum has a fixed order: the gradients are deterministic.
#include <type_traits>

#include "common.cuh"
#include "plan.h"
#include "sm100.cuh"
#include "tc.h"

namespace rece {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float2 load_pair(const float* p) {
  return *reinterpret_cast<const float2*>(p);
}
__device__ __forceinline__ float2 load_pair(const __nv_bfloat16* p) {
  const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// The coefficient's probability term: the softmax exp(l - lse) of the reduced loss and of
// CE-, or the sigmoid of BCE+ (its g is sigmoid(l) - [positive] likewise).
__device__ __forceinline__ float coef_p(float l, float li, bool sigmoid) {
  return sigmoid ? 1.0f / (1.0f + expf(-l)) : expf(l - li);
}

// <x, y> with x in shared memory (fp32) and y a catalogue row, t ascending.
template <typename T>
__device__ __forceinline__ float dot_row(const float* xs, const T* __restrict__ y, int d) {
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

// One warp per row; shared memory per warp: x (d floats), g and item of every slot.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_bwd_rows(
    const T* __restrict__ X, const T* __restrict__ Y, const int32_t* __restrict__ targets,
    const int32_t* __restrict__ selected, const float* __restrict__ lse,
    const float* __restrict__ logits, const float* __restrict__ dloss, int64_t N, int64_t C,
    int d, int k, int32_t* __restrict__ e_key, float* __restrict__ e_g, float* __restrict__ dX,
    uint32_t* status, bool sigmoid) {
  extern __shared__ __align__(16) float sh_f[];
  const int warps = blockDim.x >> 5, wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slots = k + 1;
  const int per_warp = d + 2 * slots;
  float* xs = sh_f + size_t(per_warp) * wid;
  float* gs = xs + d;
  int32_t* js = reinterpret_cast<int32_t*>(gs + slots);
  const int64_t i = int64_t(blockIdx.x) * warps + wid;
  if (i >= N) return;  // the warp leaves together; no block-wide barrier follows
  const float scale = dloss[0] / float(N);
  const float li = sigmoid ? 0.0f : lse[i];
  if (!logits)  // x takes part only in the dot products
    for (int t = lane; t < d; t += 32) xs[t] = to_f32(X[i * d + t]);
  __syncwarp();

  // coefficients: one slot per lane at a time
  for (int s = lane; s < slots; s += 32) {
    int32_t j = s == 0 ? targets[i] : selected[i * k + (s - 1)];
    float g = 0.0f;
    if (j >= 0 && j < C) {
      const float l = logits ? logits[i * slots + s] : dot_row(xs, Y + int64_t(j) * d, d);
      const float p = coef_p(l, li, sigmoid);
      g = (s == 0 ? p - 1.0f : p) * scale;
    } else {
      if (s == 0) raise_flag(status, RECE_DEVICE_BAD_TARGET);
      j = -1;
    }
    gs[s] = g;
    js[s] = j;
    e_key[i * slots + s] = j < 0 ? int32_t(C) : j;
    e_g[i * slots + s] = g;
  }
  __syncwarp();

  // dX_i: lanes over dimensions (two each), slots in order
  if (!dX) return;  // dX comes from the tensor cores
  if ((d & 1) == 0) {
    for (int t0 = 0; t0 < d; t0 += 64) {
      const int t = t0 + 2 * lane;
      float a0 = 0.0f, a1 = 0.0f;
      if (t < d) {
#pragma unroll 4
        for (int s = 0; s < slots; ++s) {
          const int32_t j = js[s];
          if (j < 0) continue;
          const float g = gs[s];
          const float2 y = load_pair(Y + int64_t(j) * d + t);
          a0 = fmaf(g, y.x, a0);
          a1 = fmaf(g, y.y, a1);
        }
        *reinterpret_cast<float2*>(dX + i * d + t) = make_float2(a0, a1);
      }
    }
  } else {
    for (int t = lane; t < d; t += 32) {
      float a = 0.0f;
      for (int s = 0; s < slots; ++s) {
        const int32_t j = js[s];
        if (j >= 0) a = fmaf(gs[s], to_f32(Y[int64_t(j) * d + t]), a);
      }
      dX[i * d + t] = a;
    }
  }
}

// One warp per item: dY_j = sum over its pairs (row order) of g * x_row.  The pairs are
// read 32 at a time (entry id and g, contiguous), then broadcast one by one.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_bwd_items(
    const T* __restrict__ X, int64_t C, int d, int k, const int32_t* __restrict__ item_start,
    const int32_t* __restrict__ sorted_id, const float* __restrict__ pair_g,
    const float* __restrict__ sorted_g, float* __restrict__ dY) {
  const int lane = threadIdx.x & 31;
  const int64_t j = int64_t(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  if (j >= C) return;
  const int64_t lo = item_start[j], hi = item_start[j + 1];
  const int slots = k + 1;
  const bool pairs = (d & 1) == 0;
  const int step = pairs ? 64 : 32;
  for (int t0 = 0; t0 < d; t0 += step) {
    const int t = pairs ? t0 + 2 * lane : t0 + lane;
    float a0 = 0.0f, a1 = 0.0f;
    for (int64_t b = lo; b < hi; b += 32) {
      const int n = int(hi - b < 32 ? hi - b : 32);
      int32_t row = 0;
      float g = 0.0f;
      if (lane < n) {
        const int32_t id = sorted_id[b + lane];
        row = id / slots;
        g = sorted_g ? sorted_g[b + lane] : pair_g[id];
      }
#pragma unroll 4
      for (int q = 0; q < n; ++q) {
        const int32_t r = __shfl_sync(0xFFFFFFFFu, row, q);
        const float gq = __shfl_sync(0xFFFFFFFFu, g, q);
        if (t < d) {
          if (pairs) {
            const float2 x = load_pair(X + int64_t(r) * d + t);
            a0 = fmaf(gq, x.x, a0);
            a1 = fmaf(gq, x.y, a1);
          } else {
            a0 = fmaf(gq, to_f32(X[int64_t(r) * d + t]), a0);
          }
        }
      }
    }
    if (t < d) {
      if (pairs) *reinterpret_cast<float2*>(dY + j * d + t) = make_float2(a0, a1);
      else dY[j * d + t] = a0;
    }
  }
}

// ---------------------------------------------------------------- d % 8 == 0 kernels
// Eight lanes (a "quarter" of the warp) share one catalogue / input row: lane `sub` of
// quarter q covers dims 8*sub + 64*m, one 16-byte vector (bf16) or two (fp32) each, so a
// warp-wide load touches four whole rows.  The quarters take every fourth slot / pair and
// are added at the end in a fixed order (q0+q1)+(q2+q3): still deterministic.

template <typename T>
__device__ __forceinline__ void load8v(const T* p, float (&v)[8]) { load8(p, v); }

// One warp per row.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_bwd_rows_v8(
    const T* __restrict__ X, const T* __restrict__ Y, const int32_t* __restrict__ targets,
    const int32_t* __restrict__ selected, const float* __restrict__ lse,
    const float* __restrict__ logits, const float* __restrict__ dloss, int64_t N, int64_t C,
    int d, int k, int32_t* __restrict__ e_key, float* __restrict__ e_g, float* __restrict__ dX,
    uint32_t* status, bool sigmoid) {
  extern __shared__ __align__(16) float sh_f[];
  const int warps = blockDim.x >> 5, wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = lane >> 3, sub = lane & 7;
  const int slots = k + 1;
  const int per_warp = d + 2 * slots;
  float* xs = sh_f + size_t(per_warp) * wid;
  float* gs = xs + d;
  int32_t* js = reinterpret_cast<int32_t*>(gs + slots);
  const int64_t i = int64_t(blockIdx.x) * warps + wid;
  if (i >= N) return;  // the warp leaves together; no block-wide barrier follows
  const float scale = dloss[0] / float(N);
  const float li = sigmoid ? 0.0f : lse[i];
  if (!logits)  // x takes part only in the dot products
    for (int t = lane; t < d; t += 32) xs[t] = to_f32(X[i * d + t]);
  __syncwarp();

  if (logits) {
    // the forward's logits: no dot products; one slot per lane
    for (int s = lane; s < slots; s += 32) {
      int32_t j = s == 0 ? targets[i] : selected[i * k + (s - 1)];
      const bool ok = j >= 0 && j < C;
      float g = 0.0f;
      if (ok) {
        const float p = coef_p(logits[i * slots + s], li, sigmoid);
        g = (s == 0 ? p - 1.0f : p) * scale;
      } else if (s == 0) {
        raise_flag(status, RECE_DEVICE_BAD_TARGET);
      }
      gs[s] = g;
      js[s] = ok ? j : -1;
      e_key[i * slots + s] = ok ? j : int32_t(C);
      e_g[i * slots + s] = g;
    }
  }
  // coefficients: sixteen slots per step, four per quarter, their rows loaded together
  for (int s0 = 0; s0 < (logits ? 0 : slots); s0 += 16) {
    int32_t j[4];
    bool ok[4];
    float part[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int s = s0 + 4 * u + q;
      j[u] = -1;
      if (s < slots) j[u] = s == 0 ? targets[i] : selected[i * k + (s - 1)];
      ok[u] = j[u] >= 0 && j[u] < C;
      part[u] = 0.0f;
    }
    for (int t = 8 * sub; t < d; t += 64) {
      float v[4][8];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (ok[u]) load8v(Y + int64_t(j[u]) * d + t, v[u]);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (ok[u]) {
#pragma unroll
          for (int uu = 0; uu < 8; ++uu) part[u] = fmaf(xs[t + uu], v[u][uu], part[u]);
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      part[u] += __shfl_xor_sync(0xFFFFFFFFu, part[u], 4);
      part[u] += __shfl_xor_sync(0xFFFFFFFFu, part[u], 2);
      part[u] += __shfl_xor_sync(0xFFFFFFFFu, part[u], 1);
    }
    if (sub == 0) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int s = s0 + 4 * u + q;
        if (s >= slots) continue;
        float g = 0.0f;
        if (ok[u]) {
          const float p = coef_p(part[u], li, sigmoid);
          g = (s == 0 ? p - 1.0f : p) * scale;
        } else if (s == 0) {
          raise_flag(status, RECE_DEVICE_BAD_TARGET);
        }
        gs[s] = g;
        js[s] = ok[u] ? j[u] : -1;
        e_key[i * slots + s] = ok[u] ? j[u] : int32_t(C);
        e_g[i * slots + s] = g;
      }
    }
  }
  __syncwarp();

  // dX_i: quarter q adds the slots s = q (mod 4) in order over its lane's 8 dims (not
  // here when dX comes from the tensor cores)
  for (int t0 = 0; t0 < (dX ? d : 0); t0 += 64) {
    const int t = t0 + 8 * sub;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (t < d) {
      for (int s = q; s < slots; s += 16) {
        float v[4][8];
        float g[4];
        bool has[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int su = s + 4 * u;
          const int32_t j = su < slots ? js[su] : -1;
          has[u] = j >= 0;
          g[u] = has[u] ? gs[su] : 0.0f;
          if (has[u]) load8v(Y + int64_t(j) * d + t, v[u]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (has[u]) {
#pragma unroll
            for (int uu = 0; uu < 8; ++uu) acc[uu] = fmaf(g[u], v[u][uu], acc[uu]);
          }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      acc[u] += __shfl_xor_sync(0xFFFFFFFFu, acc[u], 8);
      acc[u] += __shfl_xor_sync(0xFFFFFFFFu, acc[u], 16);
    }
    if (q == 0 && t < d) {
      float4* o = reinterpret_cast<float4*>(dX + i * d + t);
      o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

// One warp per item; quarter q adds the pairs b = lo + q (mod 4) in row order.  With
// `long_items`, an item of more than kLongRunPairs pairs is only listed there (count in
// long_items[0]) for k_bwd_items_long.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_bwd_items_v8(
    const T* __restrict__ X, int64_t C, int d, int k, const int32_t* __restrict__ item_start,
    const int32_t* __restrict__ sorted_id, const float* __restrict__ pair_g,
    const float* __restrict__ sorted_g, int32_t* __restrict__ long_items,
    float* __restrict__ dY) {
  const int lane = threadIdx.x & 31, q = lane >> 3, sub = lane & 7;
  const int64_t j = int64_t(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  if (j >= C) return;
  const int64_t lo = item_start[j], hi = item_start[j + 1];
  if (long_items && hi - lo > kLongRunPairs) {  // a popular item: k_bwd_items_long sums it
    if (lane == 0) long_items[1 + atomicAdd(long_items, 1)] = int32_t(j);
    return;
  }
  const int slots = k + 1;
  for (int t0 = 0; t0 < d; t0 += 64) {
    const int t = t0 + 8 * sub;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int64_t b = lo; b < hi; b += 32) {
      const int n = int(hi - b < 32 ? hi - b : 32);
      int32_t row = 0;
      float g = 0.0f;
      if (lane < n) {
        const int32_t id = sorted_id[b + lane];
        row = id / slots;
        g = sorted_g ? sorted_g[b + lane] : pair_g[id];
      }
      for (int e0 = 0; e0 < n; e0 += 4) {
        const int e = e0 + q;
        const int32_t r = __shfl_sync(0xFFFFFFFFu, row, e & 31);
        const float ge = __shfl_sync(0xFFFFFFFFu, g, e & 31);
        if (e < n && t < d) {
          float v[8];
          load8v(X + int64_t(r) * d + t, v);
#pragma unroll
          for (int u = 0; u < 8; ++u) acc[u] = fmaf(ge, v[u], acc[u]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      acc[u] += __shfl_xor_sync(0xFFFFFFFFu, acc[u], 8);
      acc[u] += __shfl_xor_sync(0xFFFFFFFFu, acc[u], 16);
    }
    if (q == 0 && t < d) {
      float4* o = reinterpret_cast<float4*>(dY + j * d + t);
      o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

// dY of the items k_bwd_items_v8 left out (runs of more than kLongRunPairs pairs: the
// targets are Zipf-drawn, and the most popular item's run would keep one warp busy long
// after the others finished).  A CTA per listed item: warp w sums the w-th of kLongWarps
// contiguous parts of the run (pairs in order, four rows in flight, as k_bwd_items_v8),
// then one thread per dimension adds the warps' parts in warp order: deterministic.
// long_items[0] is the count, the ids follow (their order does not matter: each item is
// summed by one CTA alone).
constexpr int kLongWarps = 16;

template <typename T>
__global__ void __launch_bounds__(kLongWarps * 32) k_bwd_items_long(
    const T* __restrict__ X, int d, int k, const int32_t* __restrict__ item_start,
    const int32_t* __restrict__ sorted_id, const float* __restrict__ pair_g,
    const float* __restrict__ sorted_g, const int32_t* __restrict__ long_items,
    float* __restrict__ dY) {
  __shared__ float part[kLongWarps][64];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, q = lane >> 3, sub = lane & 7;
  const int count = long_items[0];
  const int slots = k + 1;
  for (int li = blockIdx.x; li < count; li += gridDim.x) {
    const int64_t j = long_items[1 + li];
    const int64_t lo = item_start[j], n = item_start[j + 1] - lo;
    const int64_t a0 = lo + n * warp / kLongWarps, a1 = lo + n * (warp + 1) / kLongWarps;
    for (int t0 = 0; t0 < d; t0 += 64) {
      const int t = t0 + 8 * sub;
      float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int64_t b = a0; b < a1; b += 32) {
        const int m = int(a1 - b < 32 ? a1 - b : 32);
        int32_t row = 0;
        float g = 0.0f;
        if (lane < m) {
          const int32_t id = sorted_id[b + lane];
          row = id / slots;
          g = sorted_g ? sorted_g[b + lane] : pair_g[id];
        }
        for (int e0 = 0; e0 < m; e0 += 4) {
          const int e = e0 + q;
          const int32_t r = __shfl_sync(0xFFFFFFFFu, row, e & 31);
          const float ge = __shfl_sync(0xFFFFFFFFu, g, e & 31);
          if (e < m && t < d) {
            float v[8];
            load8v(X + int64_t(r) * d + t, v);
#pragma unroll
            for (int u = 0; u < 8; ++u) acc[u] = fmaf(ge, v[u], acc[u]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        acc[u] += __shfl_xor_sync(0xFFFFFFFFu, acc[u], 8);
        acc[u] += __shfl_xor_sync(0xFFFFFFFFu, acc[u], 16);
      }
      __syncthreads();  // the last slice's parts are added
      if (q == 0) {
#pragma unroll
        for (int u = 0; u < 8; ++u) part[warp][8 * sub + u] = acc[u];
      }
      __syncthreads();
      if (threadIdx.x < 64 && t0 + int(threadIdx.x) < d) {
        float s = 0.0f;
        for (int w = 0; w < kLongWarps; ++w) s += part[w][threadIdx.x];
        dY[j * d + t0 + threadIdx.x] = s;
      }
    }
  }
}

// dY for wide rows (1024 <= d <= 4096, d % 16 == 0): one CTA per item.  Warp 0 streams
// the item's pairs' x rows, each one contiguous bulk copy, through a ring of shared-memory
// stages; every other thread owns 16 dimensions and adds g * x for each pair in order.
// The rows reach the SM without passing through registers, so far more bytes are in
// flight than a register-gathering warp can hold.  Each dimension is summed by one
// thread in the pairs' (row) order: deterministic.  Waits are bounded; a timeout sets
// the device flag and ends the CTA's work.
constexpr int kWideMaxStages = 8;
constexpr uint64_t kWideTimeoutNs = 1000000000ull;

int wide_stages(int d, size_t elem) {
  const size_t rb = size_t(d) * elem;
  int st = int((64 * 1024) / rb);
  return st < 2 ? 2 : (st > kWideMaxStages ? kWideMaxStages : st);
}

template <typename T>
__global__ void __launch_bounds__(288) k_bwd_items_wide(
    const T* __restrict__ X, int d, int k, int stages, const int32_t* __restrict__ item_start,
    const int32_t* __restrict__ sorted_id, const float* __restrict__ pair_g,
    const float* __restrict__ sorted_g, float* __restrict__ dY, uint32_t* status) {
  extern __shared__ __align__(128) uint8_t wsm[];
  __shared__ uint64_t full[kWideMaxStages], empty[kWideMaxStages];
  __shared__ float s_g[kWideMaxStages];
  __shared__ int abort_flag;
  const uint32_t rb = uint32_t(d) * sizeof(T);
  const int64_t j = blockIdx.x;
  const int64_t lo = item_start[j];
  const int n = int(item_start[j + 1] - lo);
  const int consumers = (blockDim.x >> 5) - 1;  // warps
  if (n == 0) {  // an item no pair names: zeros, without setting up the ring
    if (threadIdx.x >= 32) {
      float4* o = reinterpret_cast<float4*>(dY + j * d + (threadIdx.x - 32) * 16);
#pragma unroll
      for (int e = 0; e < 4; ++e) __stcs(o + e, make_float4(0.0f, 0.0f, 0.0f, 0.0f));
    }
    return;
  }
  if (threadIdx.x == 0) {
    for (int st = 0; st < stages; ++st) {
      sm100::mbar_init(&full[st], 1);
      sm100::mbar_init(&empty[st], consumers);
    }
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    // ------------------------------------------------------------ producer
    if (threadIdx.x == 0) {
      const int slots = k + 1;
      int q = 0;
      for (; q < n; ++q) {
        const int st = q % stages;
        if (q >= stages &&
            !sm100::mbar_wait(&empty[st], uint32_t((q / stages) - 1) & 1u, &abort_flag,
                              kWideTimeoutNs)) {
          abort_flag = 1;
          raise_flag(status, RECE_DEVICE_TIMEOUT);
          break;
        }
        const int32_t id = sorted_id[lo + q];
        s_g[st] = sorted_g ? sorted_g[lo + q] : pair_g[id];
        sm100::mbar_arrive_expect_tx(&full[st], rb);
        sm100::bulk_load(wsm + size_t(st) * rb, X + int64_t(id / slots) * d, rb, &full[st]);
      }
      // every issued copy has landed before the CTA may exit
      for (int p = (q > stages ? q - stages : 0); p < q; ++p)
        sm100::mbar_wait_limit(&full[p % stages], uint32_t(p / stages) & 1u, kWideTimeoutNs);
    }
    return;
  }
  // -------------------------------------------------------------- consumers
  const int t0 = (threadIdx.x - 32) * 16;
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
  for (int q = 0; q < n; ++q) {
    const int st = q % stages;
    if (!sm100::mbar_wait(&full[st], uint32_t(q / stages) & 1u, &abort_flag, kWideTimeoutNs)) {
      abort_flag = 1;
      raise_flag(status, RECE_DEVICE_TIMEOUT);
      break;
    }
    const T* row = reinterpret_cast<const T*>(wsm + size_t(st) * rb) + t0;
    const float g = s_g[st];
    float v[16];
    load8(row, *reinterpret_cast<float(*)[8]>(&v[0]));
    load8(row + 8, *reinterpret_cast<float(*)[8]>(&v[8]));
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = fmaf(g, v[e], acc[e]);
    __syncwarp();
    if ((threadIdx.x & 31) == 0) sm100::mbar_arrive(&empty[st]);
  }
  // streaming stores: dY is written once, and should not push the gathered rows of X
  // out of L2
  float4* o = reinterpret_cast<float4*>(dY + j * d + t0);
#pragma unroll
  for (int e = 0; e < 4; ++e)
    __stcs(o + e, make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]));
}

// The run of equal keys holding position p: run_lo[p] its first position, run_hi[p] the
// first past it (two binary searches per position).
__global__ void __launch_bounds__(256) k_runs(const int32_t* __restrict__ key, int64_t E,
                                              int32_t* __restrict__ run_lo,
                                              int32_t* __restrict__ run_hi) {
  const int64_t p = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (p >= E) return;
  const int32_t j = key[p];
  int64_t lo = 0, hi = p;
  while (lo < hi) {
    const int64_t mid = (lo + hi) >> 1;
    if (key[mid] < j) lo = mid + 1;
    else hi = mid;
  }
  run_lo[p] = int32_t(lo);
  lo = p + 1;
  hi = E;
  while (lo < hi) {
    const int64_t mid = (lo + hi) >> 1;
    if (key[mid] <= j) lo = mid + 1;
    else hi = mid;
  }
  run_hi[p] = int32_t(lo);
}

constexpr int kSeg = 32;  // pairs per segment of a run

// The positives' terms of dY, in two levels so that a popular target's long run (the
// targets are Zipf-drawn) is summed in parallel.  Level 1: one warp per (segment of up to
// 32 pairs of a run, 256 columns of d), eight pairs' rows in flight, pairs in order; a run
// of one segment adds its sum into the item's row, a longer run leaves each segment's sum
// in part[first position of the segment].  Level 2 (k_pos_dy_runs): the run's first
// position adds the parts into eight partial sums (part u, u + 8, ...) and those in a
// fixed tree.  Deterministic.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_pos_dy_seg(
    const T* __restrict__ X, int64_t C, int d, int slots, const int32_t* __restrict__ key,
    const int32_t* __restrict__ run_lo, const int32_t* __restrict__ run_hi,
    const int32_t* __restrict__ sorted_id, const float* __restrict__ pair_g, int64_t E,
    float* __restrict__ part, float* __restrict__ dY) {
  const int lane = threadIdx.x & 31;
  const int64_t p = int64_t(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  if (p >= E) return;
  const int32_t j = key[p];
  const int64_t r0 = run_lo[p], r1 = run_hi[p];
  if (j >= C || (p - r0) % kSeg != 0) return;
  const int t0 = blockIdx.y * 256 + 8 * lane;
  if (t0 >= d) return;
  const int64_t q1 = p + kSeg < r1 ? p + kSeg : r1;
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int64_t q = p; q < q1; q += 8) {
    float v[8][8], gq[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      gq[u] = 0.0f;
      if (q + u < q1) {
        const int32_t id = sorted_id[q + u];
        gq[u] = pair_g[id];
        load8(X + int64_t(id / slots) * d + t0, v[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (q + u < q1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(gq[u], v[u][e], acc[e]);
      }
  }
  float4* o = reinterpret_cast<float4*>(r1 - r0 <= kSeg ? dY + int64_t(j) * d + t0
                                                         : part + p * d + t0);
  if (r1 - r0 <= kSeg) {
    float4 a0 = o[0], a1 = o[1];
    a0.x += acc[0]; a0.y += acc[1]; a0.z += acc[2]; a0.w += acc[3];
    a1.x += acc[4]; a1.y += acc[5]; a1.z += acc[6]; a1.w += acc[7];
    o[0] = a0;
    o[1] = a1;
  } else {
    o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

__global__ void __launch_bounds__(kThreads) k_pos_dy_runs(
    int64_t C, int d, const int32_t* __restrict__ key, const int32_t* __restrict__ run_lo,
    const int32_t* __restrict__ run_hi, int64_t E, const float* __restrict__ part,
    float* __restrict__ dY) {
  const int lane = threadIdx.x & 31;
  const int64_t p = int64_t(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  if (p >= E) return;
  const int32_t j = key[p];
  const int64_t r1 = run_hi[p];
  if (j >= C || run_lo[p] != p || r1 - p <= kSeg) return;
  // eight parts' loads in flight at a time, into eight partial sums added in a fixed tree
  // (a Zipf-drawn target's run holds thousands of positives: hundreds of parts)
  for (int t = blockIdx.y * 256 + lane; t < d && t < int(blockIdx.y + 1) * 256; t += 32) {
    float s[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    int64_t q = p;
    for (; q + 7 * kSeg < r1; q += 8 * kSeg) {
#pragma unroll
      for (int u = 0; u < 8; ++u) s[u] += part[(q + u * kSeg) * d + t];
    }
    for (; q < r1; q += kSeg) s[0] += part[q * d + t];
    dY[int64_t(j) * d + t] += ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
  }
}

}  // namespace

size_t bwd_rows_warp_bytes(int d, int k) { return sizeof(float) * size_t(d + 2 * (k + 1)); }

// LSD radix sort of E pairs by item key (values 0..C), as few passes as the counting
// sort's 12-bit digit limit allows.  Every pass writes the keys (and g, when given) in its
// output order, so the next pass reads them contiguously; *sorted_id (perm_a or perm_b)
// says where each sorted pair came from.  The last pass lands in sorted_key / sorted_g.
cudaError_t sort_pairs_by_item(const rece_plan_s& p, int64_t E, const int32_t* key,
                               const float* g, int32_t* perm_a, int32_t* perm_b, int32_t* key_b,
                               float* g_b, int32_t* sorted_key, float* sorted_g, void* scratch,
                               const int32_t** sorted_id, cudaStream_t st) {
  int32_t* key_buf[2] = {key_b, sorted_key};
  float* g_buf[2] = {g_b, sorted_g};
  const int passes = p.item_passes;
  const int32_t* in = nullptr;
  const int32_t* kin = key;
  const float* gin = g;
  int32_t* out = perm_a;
  int shift = 0;
  for (int ps = 0; ps < passes; ++ps) {
    const int bits = (ps + 1 < passes) ? p.item_pass_bits : p.item_bits - shift;
    const int slot = (passes - 1 - ps) % 2 == 0 ? 1 : 0;
    cudaError_t e = launch_sort_pass(kin, in, E, shift, bits, scratch, out, key_buf[slot],
                                     nullptr, st, gin, gin ? g_buf[slot] : nullptr, ps > 0);
    if (e != cudaSuccess) return e;
    shift += bits;
    in = out;
    kin = key_buf[slot];
    gin = gin ? g_buf[slot] : nullptr;
    out = (out == perm_a) ? perm_b : perm_a;
  }
  *sorted_id = in;
  return cudaSuccess;
}

template <typename T>
cudaError_t launch_backward(const rece_plan_s& p, const T* X, const T* Y,
                            const int32_t* targets, const int32_t* selected, const float* lse,
                            const float* logits, const float* dloss, char* ws, float* dX,
                            float* dY, uint32_t* status, cudaStream_t st) {
  // with dX on the tensor cores the rows kernel only lays out the (item, g) pairs
  bool dx_tc = false;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) dx_tc = p.tc_dx;
  const auto& c = p.cfg;
  const Layout& L = p.lay;
  const int64_t E = p.entries;
  int32_t* e_key = reinterpret_cast<int32_t*>(ws + L.e_key);
  float* e_g = reinterpret_cast<float*>(ws + L.e_g);
  int32_t* perm_a = reinterpret_cast<int32_t*>(ws + L.e_perm_a);
  int32_t* perm_b = reinterpret_cast<int32_t*>(ws + L.e_perm_b);
  int32_t* sorted_key = reinterpret_cast<int32_t*>(ws + L.e_sorted_key);
  float* sorted_g = p.carry_g ? reinterpret_cast<float*>(ws + L.e_sorted_g) : nullptr;
  void* scratch = ws + L.e_scratch;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    if (p.tc_dy) {
      // dX and dY as band products on the tensor cores (dY written by round 0, added by
      // the others), then the positives' dY terms added from their sorted pairs
      stage_mark(p, RECE_STAGE_BWD_ROWS, 0, st);
      cudaError_t e = launch_dx_tc(p, Y, targets, lse, dloss, ws, dX, status, st);
      if (e != cudaSuccess) return e;
      stage_mark(p, RECE_STAGE_BWD_ROWS, 1, st);
      stage_mark(p, RECE_STAGE_BWD_ITEMS, 0, st);
      e = launch_dy_tc(p, dloss, ws, dY, status, st);
      if (e != cudaSuccess) return e;
      stage_mark(p, RECE_STAGE_BWD_ITEMS, 1, st);
      stage_mark(p, RECE_STAGE_BWD_SORT, 0, st);
      const rece_plan_s& q = *p.pos_plan;  // k = 0: one slot per row, its positive
      if (c.N > 0) {
        const size_t per_warp = bwd_rows_warp_bytes(c.d, 0);
        int warps = int((200 * 1024) / per_warp);
        warps = warps < 1 ? 1 : (warps > kThreads / 32 ? kThreads / 32 : warps);
        // the merge stored each row's positive logit: a k = 0 plan's logits [N][1]
        const float* plog = reinterpret_cast<const float*>(ws + L.pos_logit);
        e = cudaFuncSetAttribute(k_bwd_rows_v8<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(per_warp * warps));
        if (e != cudaSuccess) return e;
        k_bwd_rows_v8<T><<<unsigned(ceil_div(c.N, warps)), warps * 32, per_warp * warps, st>>>(
            X, Y, targets, selected, lse, plog, dloss, c.N, c.C, c.d, 0, e_key, e_g, nullptr,
            status, false);
        count_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int32_t* in = nullptr;
        e = sort_pairs_by_item(q, c.N, e_key, nullptr, perm_a, perm_b,
                               reinterpret_cast<int32_t*>(ws + L.e_key_b), nullptr, sorted_key,
                               nullptr, scratch, &in, st);
        if (e != cudaSuccess) return e;
        // the runs of equal targets, in the arrays the sort no longer needs
        int32_t* run_lo = reinterpret_cast<int32_t*>(ws + L.e_key_b);
        int32_t* run_hi = const_cast<int32_t*>(in) == perm_a ? perm_b : perm_a;
        float* part = reinterpret_cast<float*>(ws + L.pos_parts);
        const dim3 grid(unsigned(ceil_div(c.N, kThreads / 32)), unsigned(ceil_div(c.d, 256)));
        k_runs<<<unsigned(ceil_div(c.N, 256)), 256, 0, st>>>(sorted_key, c.N, run_lo, run_hi);
        k_pos_dy_seg<T><<<grid, kThreads, 0, st>>>(X, c.C, c.d, 1, sorted_key, run_lo, run_hi,
                                                   in, e_g, c.N, part, dY);
        k_pos_dy_runs<<<grid, kThreads, 0, st>>>(c.C, c.d, sorted_key, run_lo, run_hi, c.N,
                                                 part, dY);
        count_launches(3);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
      }
      stage_mark(p, RECE_STAGE_BWD_SORT, 1, st);
      return cudaSuccess;
    }
  }
  stage_mark(p, RECE_STAGE_BWD_ROWS, 0, st);
  if (c.N > 0) {
    const size_t per_warp = bwd_rows_warp_bytes(c.d, c.k);
    int warps = int((200 * 1024) / per_warp);
    warps = warps < 1 ? 1 : (warps > kThreads / 32 ? kThreads / 32 : warps);
    const size_t smem = per_warp * warps;
    const bool v8 = (c.d % 8) == 0;
    cudaError_t e = cudaFuncSetAttribute(v8 ? k_bwd_rows_v8<T> : k_bwd_rows<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    float* dx_rows = dx_tc ? nullptr : dX;
    if (v8)
      k_bwd_rows_v8<T><<<unsigned(ceil_div(c.N, warps)), warps * 32, smem, st>>>(
          X, Y, targets, selected, lse, logits, dloss, c.N, c.C, c.d, c.k, e_key, e_g, dx_rows,
          status, p.sigmoid_g);
    else
      k_bwd_rows<T><<<unsigned(ceil_div(c.N, warps)), warps * 32, smem, st>>>(
          X, Y, targets, selected, lse, logits, dloss, c.N, c.C, c.d, c.k, e_key, e_g, dx_rows,
          status, p.sigmoid_g);
    count_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
      if (dx_tc) {
        e = launch_dx_tc(p, Y, targets, lse, dloss, ws, dX, status, st);
        if (e != cudaSuccess) return e;
      }
    }
  }
  stage_mark(p, RECE_STAGE_BWD_ROWS, 1, st);
  stage_mark(p, RECE_STAGE_BWD_SORT, 0, st);
  const int32_t* in = nullptr;
  {
    cudaError_t e = sort_pairs_by_item(
        p, E, e_key, p.carry_g ? e_g : nullptr, perm_a, perm_b,
        reinterpret_cast<int32_t*>(ws + L.e_key_b), reinterpret_cast<float*>(ws + L.e_g_b),
        sorted_key, sorted_g, scratch, &in, st);
    if (e != cudaSuccess) return e;
  }
  int32_t* item_start = reinterpret_cast<int32_t*>(ws + L.e_item_start);
  cudaError_t e2 = launch_segment_starts(sorted_key, E, int32_t(c.C), item_start, st);
  if (e2 != cudaSuccess) return e2;
  stage_mark(p, RECE_STAGE_BWD_SORT, 1, st);
  stage_mark(p, RECE_STAGE_BWD_ITEMS, 0, st);
  const int warps = kThreads / 32;
  if (c.d >= 1024 && c.d <= 4096 && c.d % 16 == 0) {
    const int stages = wide_stages(c.d, sizeof(T));
    const size_t smem = size_t(stages) * c.d * sizeof(T);
    cudaError_t e = cudaFuncSetAttribute(k_bwd_items_wide<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    k_bwd_items_wide<T><<<unsigned(c.C), 32 + c.d / 16, smem, st>>>(
        X, c.d, c.k, stages, item_start, in, e_g, sorted_g, dY, status);
  } else if (c.d % 8 == 0) {
    // popular items go to a list that k_bwd_items_long sums, a CTA per item
    int32_t* long_items = reinterpret_cast<int32_t*>(ws + L.e_long);
    cudaError_t e = cudaMemsetAsync(long_items, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return e;
    k_bwd_items_v8<T><<<unsigned(ceil_div(c.C, warps)), kThreads, 0, st>>>(
        X, c.C, c.d, c.k, item_start, in, e_g, sorted_g, long_items, dY);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_bwd_items_long<T><<<unsigned(2 * sm_count()), kLongWarps * 32, 0, st>>>(
        X, c.d, c.k, item_start, in, e_g, sorted_g, long_items, dY);
  } else
    k_bwd_items<T><<<unsigned(ceil_div(c.C, warps)), kThreads, 0, st>>>(
        X, c.C, c.d, c.k, item_start, in, e_g, sorted_g, dY);
  count_launches(1);
  stage_mark(p, RECE_STAGE_BWD_ITEMS, 1, st);
  return cudaGetLastError();
}

template cudaError_t launch_backward<float>(const rece_plan_s&, const float*, const float*,
                                            const int32_t*, const int32_t*, const float*,
                                            const float*, const float*, char*, float*, float*,
                                            uint32_t*, cudaStream_t);
template cudaError_t launch_backward<__nv_bfloat16>(const rece_plan_s&, const __nv_bfloat16*,
                                                    const __nv_bfloat16*, const int32_t*,
                                                    const int32_t*, const float*, const float*,
                                                    const float*, char*, float*, float*,
                                                    uint32_t*, cudaStream_t);

}  // namespace rece
