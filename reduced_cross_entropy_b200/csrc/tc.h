// tc.h -- internal interface of the tcgen05 (tensor-core) kernels of the bf16 mode.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "plan.h"

namespace rece {

// Tensor map of a row-major bf16 matrix [rows x cols] (cols a multiple of 64), boxes of
// 64 columns x box_rows rows, 128-byte swizzle (the K-major layout the MMA reads).
cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows);
int sm_count();

// bf16 mode without RECE_FLAG_FMA_SCORES and d a multiple of 64: the tcgen05 kernels run.
bool tc_supported(const rece_plan_s& p);

// K1 on tensor cores: bucket[r][i] = argmax_b <B[r][b], V[i]> for V = X and V = Y.
cudaError_t launch_bucketize_tc(const rece_plan_s& p, const void* X, const void* Y,
                                const void* B, int32_t* bx, int32_t* by, uint32_t* status,
                                cudaStream_t st);

// Sorted row copies (bf16) and inverse orders / per-round chunk of every row.
cudaError_t launch_permute_rows(const void* V, int64_t M, int d, const int32_t* perm, int n_r,
                                int n_c, void* Vs, int32_t* inv, int32_t* chunk,
                                cudaStream_t st);

// K3 on tensor cores: per (round, sorted row) the candidate list (score bits, sorted
// catalogue position), its count and threshold.
int tc_list_capacity(int k);      // entries per (round, row): 4 sub-lists
int tc_sublist_capacity(int k);   // entries per sub-list
cudaError_t launch_select_tc(const rece_plan_s& p, const void* Xs, const void* Ys, int2* list,
                             int4* list_count, float* list_theta, uint32_t* status,
                             cudaStream_t st);

// K4 for the tensor-core lists: merge, select, order, loss, exactness check.
size_t merge_tc_warp_bytes(int n_r, int k);
template <typename T>
cudaError_t launch_merge_tc(const rece_plan_s& p, const T* X, const T* Y, const int32_t* targets,
                            const int32_t* py, const int32_t* invX, const int32_t* chunkY,
                            const int2* list, const int4* list_count,
                            const float* list_theta, int32_t* selected, float* lse,
                            float* row_loss, float* logits, uint32_t* status, cudaStream_t st);

}  // namespace rece
