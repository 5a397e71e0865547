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

}  // namespace rece
