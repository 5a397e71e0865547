// select.cu -- steps 3-4 of the path, CUDA-core version with fmaf-chain scores.
//
// RECE, section 3, Algorithm 1: the rows of sorted chunk c are scored against the items
// of chunks c-n_ec .. c+n_ec (edge windows clipped); SCE abstract: only the highest
// scores are kept.  One CTA takes G consecutive sorted rows of one chunk in one round:
//   1. every thread scores window items against the G rows (fixed-order fmaf chains),
//      writing a monotone 32-bit key per (row, item) into shared memory -- the row's
//      positive gets key 0 (never a negative);
//   2. per row, a block-wide MSB-first radix select (4 passes of 8 bits) finds the
//      k-th largest key; if the k-th place is tied, a second select on the item ids
//      keeps the lowest ids;
//   3. the k winners (score, item) go to the row's per-round list, unordered (the merge
//      kernel orders them).
// The score tile never leaves shared memory.
#include "common.cuh"
#include "plan.h"

namespace rece {
namespace {

constexpr int kThreads = 256;

// Among n elements (get(q, key) -> is element q in play, its key), find the want-th
// largest key (1 <= want <= number in play).  Returns the key value T and, through
// need/eq, how many elements equal to T belong to the top `want` and how many equal T.
template <typename Get>
__device__ void block_radix_select(int n, int want, Get get, uint32_t* hist, int* sh,
                                   uint32_t& T, int& need, int& eq) {
  uint32_t prefix = 0, pmask = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    for (int q = threadIdx.x; q < n; q += blockDim.x) {
      uint32_t key;
      if (get(q, key) && (key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      int c[8], s = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {  // lane 0 holds the 8 highest bins, highest first
        c[u] = int(hist[255 - 8 * lane - u]);
        s += c[u];
      }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
      }
      const int excl = incl - s;
      if (excl < want && want <= incl) {
        int run = excl;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (run + c[u] >= want) {
            sh[0] = 255 - 8 * lane - u;
            sh[1] = run;
            sh[2] = c[u];
            break;
          }
          run += c[u];
        }
      }
    }
    __syncthreads();
    const uint32_t digit = uint32_t(sh[0]);
    want -= sh[1];
    eq = sh[2];
    prefix |= digit << shift;
    pmask |= 0xFFu << shift;
    __syncthreads();
  }
  T = prefix;
  need = want;
}

template <typename T, int G>
__global__ void __launch_bounds__(kThreads) k_select_fma(
    const T* __restrict__ X, const T* __restrict__ Y, const int32_t* __restrict__ targets,
    const int32_t* __restrict__ px, const int32_t* __restrict__ py, int64_t N, int64_t C, int d,
    int n_c, int n_ec, int k, int groups_per_chunk, int w_max, float* __restrict__ list_score,
    int32_t* __restrict__ list_item) {
  extern __shared__ __align__(16) unsigned char sh_raw[];
  float* xs = reinterpret_cast<float*>(sh_raw);                 // [G][d]
  uint32_t* keys = reinterpret_cast<uint32_t*>(xs + G * d);     // [G][w_max]
  uint32_t* hist = keys + size_t(G) * w_max;                    // [256]
  int* sh = reinterpret_cast<int*>(hist + 256);                 // [8]
  int* row_id = sh + 8;                                         // [G]
  int* row_z = row_id + G;                                      // [G]
  int* z_in = row_z + G;                                        // [G]

  const int r = blockIdx.y;
  const int c = blockIdx.x / groups_per_chunk, gi = blockIdx.x % groups_per_chunk;
  const int64_t xs0 = chunk_start(c, N, n_c), xs1 = chunk_start(c + 1, N, n_c);
  const int64_t p0 = xs0 + int64_t(gi) * G;
  if (p0 >= xs1) return;
  const int nrows = int(xs1 - p0 < G ? xs1 - p0 : G);
  const int64_t w0 = chunk_start(max(0, c - n_ec), C, n_c);
  const int64_t w1 = chunk_start(min(n_c, c + n_ec + 1), C, n_c);
  const int W = int(w1 - w0);
  const int32_t* pyr = py + int64_t(r) * C + w0;
  const int tid = threadIdx.x;

  if (tid < G) {
    const int id = tid < nrows ? px[int64_t(r) * N + p0 + tid] : 0;
    row_id[tid] = id;
    row_z[tid] = tid < nrows ? targets[id] : -1;
    z_in[tid] = 0;
  }
  __syncthreads();
  for (int e = tid; e < G * d; e += kThreads) {
    const int g = e / d, t = e % d;
    xs[e] = g < nrows ? to_f32(X[int64_t(row_id[g]) * d + t]) : 0.0f;
  }
  __syncthreads();

  // 1. scores -> keys
  const bool vec = (d % 8) == 0;
  for (int q = tid; q < W; q += kThreads) {
    const int32_t j = pyr[q];
    const T* y = Y + int64_t(j) * d;
    float acc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g] = 0.0f;
    if (vec) {
      for (int t = 0; t < d; t += 8) {
        float yv[8];
        load8(y + t, yv);
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
          for (int g = 0; g < G; ++g) acc[g] = fmaf(xs[g * d + t + u], yv[u], acc[g]);
      }
    } else {
      for (int t = 0; t < d; ++t) {
        const float yv = to_f32(y[t]);
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] = fmaf(xs[g * d + t], yv, acc[g]);
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (g < nrows) {
        const bool pos = (j == row_z[g]);
        if (pos) z_in[g] = 1;
        keys[size_t(g) * w_max + q] = pos ? 0u : score_key(acc[g]);
      }
    }
  }
  __syncthreads();

  // 2-3. per row: select the k best and write them
  for (int g = 0; g < nrows; ++g) {
    const uint32_t* kr = keys + size_t(g) * w_max;
    const int i = row_id[g];
    const int n_valid = W - z_in[g];
    const int kk = min(k, n_valid);
    float* out_s = list_score + (int64_t(r) * N + i) * k;
    int32_t* out_i = list_item + (int64_t(r) * N + i) * k;
    if (tid == 0) sh[4] = 0;  // output slot counter
    __syncthreads();
    uint32_t Tk = 1, T2 = 0;
    bool tie_break = false;
    if (kk < n_valid && kk > 0) {
      int need, eq;
      block_radix_select(
          W, kk, [&](int q, uint32_t& key) { key = kr[q]; return true; }, hist, sh, Tk, need,
          eq);
      if (need != eq) {  // the k-th place is shared: keep the lowest item ids among ties
        tie_break = true;
        int need2, eq2;
        block_radix_select(
            W, need,
            [&](int q, uint32_t& key) {
              key = ~uint32_t(pyr[q]);
              return kr[q] == Tk;
            },
            hist, sh, T2, need2, eq2);
      }
    }
    for (int q = tid; q < W; q += kThreads) {
      const uint32_t key = kr[q];
      bool take;
      if (kk >= n_valid)
        take = key != 0u;
      else if (!tie_break)
        take = key >= Tk;
      else
        take = key > Tk || (key == Tk && ~uint32_t(pyr[q]) >= T2);
      if (take) {
        const int slot = atomicAdd(&sh[4], 1);
        out_s[slot] = key_score(key);
        out_i[slot] = pyr[q];
      }
    }
    for (int a = kk + tid; a < k; a += kThreads) {
      out_s[a] = -INFINITY;
      out_i[a] = -1;
    }
    __syncthreads();
  }
}

template <typename T, int G>
cudaError_t launch_g(const rece_plan_s& p, const T* X, const T* Y, const int32_t* targets,
                     const int32_t* px, const int32_t* py, float* ls, int32_t* li,
                     cudaStream_t st) {
  const auto& c = p.cfg;
  const int groups = int(ceil_div(p.x_chunk_max, G));
  const size_t smem = sizeof(float) * G * c.d + sizeof(uint32_t) * size_t(G) * p.w_max +
                      sizeof(uint32_t) * 256 + sizeof(int) * (8 + 3 * G);
  cudaError_t e = cudaFuncSetAttribute(k_select_fma<T, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(unsigned(c.n_c * groups), unsigned(c.n_r));
  k_select_fma<T, G><<<grid, kThreads, smem, st>>>(X, Y, targets, px, py, c.N, c.C, c.d, c.n_c,
                                                   c.n_ec, c.k, groups, int(p.w_max), ls, li);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

// Shared-memory bytes of the selection kernel for G rows per CTA.
size_t select_fma_smem_bytes(int G, int d, int64_t w_max) {
  return sizeof(float) * size_t(G) * d + sizeof(uint32_t) * size_t(G) * size_t(w_max) +
         sizeof(uint32_t) * 256 + sizeof(int) * (8 + 3 * G);
}

template <typename T>
cudaError_t launch_select_fma(const rece_plan_s& p, const T* X, const T* Y,
                              const int32_t* targets, const int32_t* px, const int32_t* py,
                              float* list_score, int32_t* list_item, cudaStream_t st) {
  if (p.cfg.N == 0) return cudaSuccess;
  switch (p.sel_rows) {
    case 8: return launch_g<T, 8>(p, X, Y, targets, px, py, list_score, list_item, st);
    case 4: return launch_g<T, 4>(p, X, Y, targets, px, py, list_score, list_item, st);
    case 2: return launch_g<T, 2>(p, X, Y, targets, px, py, list_score, list_item, st);
    default: return launch_g<T, 1>(p, X, Y, targets, px, py, list_score, list_item, st);
  }
}

template cudaError_t launch_select_fma<float>(const rece_plan_s&, const float*, const float*,
                                              const int32_t*, const int32_t*, const int32_t*,
                                              float*, int32_t*, cudaStream_t);
template cudaError_t launch_select_fma<__nv_bfloat16>(const rece_plan_s&, const __nv_bfloat16*,
                                                      const __nv_bfloat16*, const int32_t*,
                                                      const int32_t*, const int32_t*, float*,
                                                      int32_t*, cudaStream_t);

}  // namespace rece
