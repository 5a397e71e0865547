// permute.cu -- step 2's outputs in the layout the tensor-core kernels read: the rows of
// X and Y copied in bucket order (so a chunk and its window are contiguous row ranges a
// TMA box can load), the inverse orders, and the chunk of every item in every round.
//
//   Vs[r][p][:]       = V[perm[r][p]][:]                (bf16, 16-byte vector copies)
//   inv[r][perm[r][p]] = p
//   chunk[r][perm[r][p]] = chunk holding sorted position p (start of chunk c = ceil(cM/n_c))
// (Vs may be NULL: then only the inverse orders and chunks are written.)
// The backward's tensor-core products read Vs too, as MN-major operands.
#include "common.cuh"
#include "plan.h"
#include "tc.h"

namespace rece {
namespace {

__global__ void __launch_bounds__(256) k_permute_rows(const uint4* __restrict__ V, int64_t M,
                                                      int vec_per_row, const int32_t* __restrict__ perm,
                                                      int n_r, int n_c, uint4* __restrict__ Vs,
                                                      int32_t* __restrict__ inv,
                                                      int32_t* __restrict__ chunk) {
  // a warp copies kRows rows at a time, all their loads in flight before the stores
  // (one row of d <= 256 bf16 is one 16-byte vector per lane or less)
  constexpr int kRows = 4;
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  const int64_t total = int64_t(n_r) * M;
  for (int64_t w0 = (int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kRows;
       w0 < total; w0 += warps * kRows) {
    int32_t id[kRows];
#pragma unroll
    for (int u = 0; u < kRows; ++u) id[u] = w0 + u < total ? perm[w0 + u] : 0;
    if (Vs) {  // (no copy wanted: the inverse order and chunks only)
      for (int c0 = 0; c0 < vec_per_row; c0 += 32) {
        const int c = c0 + lane;
        uint4 v[kRows];
#pragma unroll
        for (int u = 0; u < kRows; ++u)
          if (w0 + u < total && c < vec_per_row) v[u] = V[int64_t(id[u]) * vec_per_row + c];
#pragma unroll
        for (int u = 0; u < kRows; ++u)
          if (w0 + u < total && c < vec_per_row) Vs[(w0 + u) * vec_per_row + c] = v[u];
      }
    }
    if (lane < kRows && w0 + lane < total) {
      const int64_t w = w0 + lane;
      const int64_t r = w / M, p = w % M;
      int32_t myid = id[0];
#pragma unroll
      for (int u = 1; u < kRows; ++u)
        if (lane == u) myid = id[u];
      if (inv) inv[r * M + myid] = int32_t(p);
      if (chunk) chunk[r * M + myid] = int32_t((p * n_c) / M);
    }
  }
}

}  // namespace

cudaError_t launch_permute_rows(const void* V, int64_t M, int d, const int32_t* perm, int n_r,
                                int n_c, void* Vs, int32_t* inv, int32_t* chunk,
                                cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const int64_t rows = int64_t(n_r) * M;
  const int64_t want = (rows + 31) / 32;  // 8 warps of 4 rows a block
  const int grid = int(want < 8 * 148 ? want : 8 * 148);
  k_permute_rows<<<grid, 256, 0, st>>>(static_cast<const uint4*>(V), M, d / 8, perm, n_r, n_c,
                                       static_cast<uint4*>(Vs), inv, chunk);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace rece
