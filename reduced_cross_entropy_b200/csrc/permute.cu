// permute.cu -- step 2's outputs in the layout the tensor-core kernels read: the rows of
// X and Y copied in bucket order (so a chunk and its window are contiguous row ranges a
// TMA box can load), the inverse orders, and the chunk of every item in every round.
//
//   Vs[r][p][:]       = V[perm[r][p]][:]                (bf16, 16-byte vector copies)
//   inv[r][perm[r][p]] = p
//   chunk[r][perm[r][p]] = chunk holding sorted position p (start of chunk c = ceil(cM/n_c))
//   VsT[r][t][p]      = Vs[r][p][t]   (the d-major copy the backward's tensor-core
//                                      products read: rows t of ld >= M elements)
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
    const uint4* src = V + int64_t(id) * vec_per_row;
    uint4* dst = Vs + w * vec_per_row;
    for (int c = lane; c < vec_per_row; c += 32) dst[c] = src[c];
    if (lane == 0) {
      if (inv) inv[r * M + id] = int32_t(p);
      if (chunk) chunk[r * M + id] = int32_t((p * n_c) / M);
    }
  }
}

// 64 sorted positions x 64 dimensions per block, through shared memory.
__global__ void __launch_bounds__(256) k_transpose_sorted(const uint16_t* __restrict__ Vs,
                                                          int64_t M, int d, int64_t ld,
                                                          uint16_t* __restrict__ VsT) {
  __shared__ uint16_t tile[64][64 + 8];
  const int r = blockIdx.z;
  const int64_t p0 = int64_t(blockIdx.x) * 64;
  const int t0 = blockIdx.y * 64;
  const uint16_t* src = Vs + (int64_t(r) * M) * d;
  for (int e = threadIdx.x; e < 64 * 8; e += blockDim.x) {
    const int pp = e >> 3, c8 = (e & 7) * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (p0 + pp < M) v = *reinterpret_cast<const uint4*>(src + (p0 + pp) * d + t0 + c8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      tile[pp][c8 + 2 * u] = uint16_t(w[u] & 0xFFFFu);
      tile[pp][c8 + 2 * u + 1] = uint16_t(w[u] >> 16);
    }
  }
  __syncthreads();
  uint16_t* dst = VsT + (int64_t(r) * d) * ld;
  for (int e = threadIdx.x; e < 64 * 8; e += blockDim.x) {
    const int tt = e >> 3, q8 = (e & 7) * 8;
    if (p0 + q8 >= M) continue;  // whole 8-run past the end (ld is a multiple of 8)
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      w[u] = uint32_t(tile[q8 + 2 * u][tt]) | (uint32_t(tile[q8 + 2 * u + 1][tt]) << 16);
    *reinterpret_cast<uint4*>(dst + int64_t(t0 + tt) * ld + p0 + q8) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace

cudaError_t launch_transpose_sorted(const void* Vs, int64_t M, int d, int n_r, int64_t ld,
                                    void* VsT, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  if (d % 64 != 0 || ld % 8 != 0 || ld < M) return cudaErrorInvalidValue;
  k_transpose_sorted<<<dim3(unsigned(ceil_div(M, 64)), unsigned(d / 64), unsigned(n_r)), 256, 0,
                       st>>>(static_cast<const uint16_t*>(Vs), M, d, ld,
                             static_cast<uint16_t*>(VsT));
  count_launches(1);
  return cudaGetLastError();
}

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
