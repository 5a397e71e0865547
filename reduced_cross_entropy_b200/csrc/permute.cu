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
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  const int64_t total = int64_t(n_r) * M;
  for (int64_t w = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); w < total;
       w += warps) {
    const int64_t r = w / M, p = w % M;
    const int32_t id = perm[w];
    if (Vs) {  // (no copy wanted: the inverse order and chunks only)
      const uint4* src = V + int64_t(id) * vec_per_row;
      uint4* dst = Vs + w * vec_per_row;
      for (int c = lane; c < vec_per_row; c += 32) dst[c] = src[c];
    }
    if (lane == 0) {
      if (inv) inv[r * M + id] = int32_t(p);
      if (chunk) chunk[r * M + id] = int32_t((p * n_c) / M);
    }
  }
}

}  // namespace

cudaError_t launch_permute_rows(const void* V, int64_t M, int d, const int32_t* perm, int n_r,
                                int n_c, void* Vs, int32_t* inv, int32_t* chunk,
                                cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const int64_t rows = int64_t(n_r) * M;
  const int64_t want = (rows + 7) / 8;
  const int grid = int(want < 8 * 148 ? want : 8 * 148);
  k_permute_rows<<<grid, 256, 0, st>>>(static_cast<const uint4*>(V), M, d / 8, perm, n_r, n_c,
                                       static_cast<uint4*>(Vs), inv, chunk);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace rece
