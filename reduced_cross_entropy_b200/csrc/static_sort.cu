// static_sort.cu -- the stable bucket sort (step 2 of the path) for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand this library a workspace: code that runs inside a
// host application which owns every byte of device memory through its own arena (a
// plugin or custom operator inside another framework, a serving process that reserves
// its memory at start-up and forbids further allocation), or a hot loop that cannot
// afford the latency and implicit synchronisation of an allocation.  For them this file
// keeps the sort's scratch -- its per-tile digit histograms and, when the caller passes
// no bucket_start buffer, the bucket starts -- in a fixed array of device memory that is
// part of the library image itself.
//
// The array is kStaticSortScratchBytes (4 MiB).  Every GPU the library is used on holds
// its own copy from the first use until the process exits.  All calls share it: two calls
// whose work overlaps on the GPU (different streams, or different host threads, without
// ordering between them) race on it.  Nothing in it has to start at zero: each call
// rewrites every histogram entry it later reads.
#include <mutex>

#include "common.cuh"
#include "plan.h"

namespace rece {
void set_last_error(const char* msg);
}  // namespace rece

namespace {

constexpr size_t kStaticSortScratchBytes = size_t(4) << 20;

static __device__ __align__(256) unsigned char g_sort_scratch[kStaticSortScratchBytes];

// Host code cannot use g_sort_scratch's name as a device address: it is a host-side
// stand-in.  The device address is looked up once per device (with that device current)
// and cached here.
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

rece_status_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    rece::set_last_error("rece_bucket_sort_static: cudaGetDevice failed");
    return RECE_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    rece::set_last_error("rece_bucket_sort_static: device ordinal above 63");
    return RECE_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_sort_scratch);
    if (e != cudaSuccess || p == nullptr) {
      rece::set_last_error("rece_bucket_sort_static: cudaGetSymbolAddress of the scratch failed");
      return RECE_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return RECE_OK;
}

}  // namespace

extern "C" rece_status_t rece_bucket_sort_static(const int32_t* bucket_ids, int64_t M,
                                                 int32_t n_b, int32_t* order,
                                                 int32_t* bucket_start, void* stream) {
  using namespace rece;
  if (M < 0 || M >= 2147483647 || n_b < 1 || n_b > (1 << kMaxDigitBits)) {
    set_last_error("rece_bucket_sort_static: M or n_b out of range");
    return RECE_ERR_INVALID_ARG;
  }
  if (M > 0 && (!bucket_ids || !order)) {
    set_last_error("rece_bucket_sort_static: NULL bucket_ids or order");
    return RECE_ERR_INVALID_ARG;
  }
  const int bits = bits_for(n_b);
  if (sort_scratch_bytes(M, bits) > kStaticSortScratchBytes) {
    set_last_error("rece_bucket_sort_static: histograms of M elements x 2^ceil(log2 n_b) "
                   "buckets exceed the 4 MiB static scratch");
    return RECE_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  rece_status_t s = scratch_address(&scratch);
  if (s != RECE_OK) return s;
  const cudaError_t e = launch_sort_pass(bucket_ids, nullptr, M, 0, bits, scratch, order,
                                         nullptr, bucket_start, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    set_last_error(cudaGetErrorName(e));
    return RECE_ERR_CUDA;
  }
  return RECE_OK;
}
