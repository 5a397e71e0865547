// tc_common.cu -- host helpers of the tensor-core kernels: TMA descriptors (tensor maps)
// for row-major bf16 matrices (2-D, or 3-D: planes of rows, one per round), the SM count
// of the current device, and the ordered sum of partial results.
#include <cudaTypedefs.h>

#include <mutex>

#include "plan.h"
#include "tc.h"

namespace rece {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if (rows == 0 || cols % 64 != 0 || (reinterpret_cast<uintptr_t>(base) & 15u) != 0)
    return cudaErrorInvalidValue;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                  strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t cols,
                              uint64_t rows, uint64_t planes, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if (rows == 0 || planes == 0 || cols % 64 != 0 || box_rows == 0 || box_rows > 256 ||
      (reinterpret_cast<uintptr_t>(base) & 15u) != 0)
    return cudaErrorInvalidValue;
  cuuint64_t dims[3] = {cols, rows, planes};
  cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_bf16_groups(CUtensorMap* map, const void* base, uint64_t cols,
                                  uint64_t groups, uint32_t group_rows, uint32_t box_rows,
                                  uint32_t box_groups) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if (groups == 0 || cols % 64 != 0 || box_rows == 0 || box_rows > group_rows ||
      box_rows > 256 || box_groups == 0 || box_groups > 256 ||
      (reinterpret_cast<uintptr_t>(base) & 15u) != 0)
    return cudaErrorInvalidValue;
  cuuint64_t dims[3] = {cols, group_rows, groups};
  cuuint64_t strides[2] = {cols * 2, uint64_t(group_rows) * cols * 2};
  cuuint32_t box[3] = {64, box_rows, box_groups};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {

__global__ void __launch_bounds__(256) k_add_parts(const float4* __restrict__ parts, int64_t n4,
                                                   int nparts, float4* __restrict__ out) {
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < n4;
       e += int64_t(gridDim.x) * blockDim.x) {
    float4 x = out[e];
    for (int z = 0; z < nparts; ++z) {
      const float4 q = parts[int64_t(z) * n4 + e];
      x.x += q.x;
      x.y += q.y;
      x.z += q.z;
      x.w += q.w;
    }
    out[e] = x;
  }
}

}  // namespace

cudaError_t launch_add_parts(const float* parts, int64_t n, int nparts, float* out,
                             cudaStream_t st) {
  if (n == 0 || nparts == 0) return cudaSuccess;
  if (n % 4 != 0) return cudaErrorInvalidValue;
  const int64_t n4 = n / 4, want = (n4 + 255) / 256;
  k_add_parts<<<unsigned(want < 8 * 148 ? want : 8 * 148), 256, 0, st>>>(
      reinterpret_cast<const float4*>(parts), n4, nparts, reinterpret_cast<float4*>(out));
  count_launches(1);
  return cudaGetLastError();
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n > 0 ? n : 148;
}

bool tc_supported(const rece_plan_s& p) {
  const auto& c = p.cfg;
  return c.mode == RECE_MODE_BF16 && !(c.flags & RECE_FLAG_FMA_SCORES) && c.d % 64 == 0 &&
         c.d <= 4096;
}

}  // namespace rece
