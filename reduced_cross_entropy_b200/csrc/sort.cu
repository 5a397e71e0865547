// sort.cu -- step 2 of the path: stable counting sort by bucket id (RECE, section 3,
// Algorithm 1: the argsort steps, read as stable), reused with 8-bit digits as the
// passes of an LSD radix sort of the backward's (item, row) pairs.
//
// One pass over M elements with b-bit digits:
//   hist     per tile of 2048 elements, the count of every digit (digit-major matrix)
//   scan     exclusive prefix over tiles for every digit, then over digits
//   scatter  every warp walks its 256 elements in order; one ballot per digit bit
//            gives every lane the mask of lanes holding its digit, so an element's rank
//            is the number of earlier elements with its digit: in earlier tiles,
//            earlier warps of its tile, earlier steps of its warp, lower lanes of its
//            step.  Stable.
// Several independent sorts (segments) of one digit width go in one launch sequence:
// blockIdx.y is the segment, blockIdx.x the tile (or digit) within it.
#include "common.cuh"
#include "plan.h"

namespace rece {
namespace {

constexpr int kWarps = kSortThreads / 32;      // 8
constexpr int kPerWarp = kSortTile / kWarps;   // 256
constexpr int kSteps = kPerWarp / 32;          // 8

__device__ __forceinline__ int32_t elem_id(const int32_t* in_ids, int64_t p) {
  return in_ids ? in_ids[p] : int32_t(p);
}
// Key (and payload) of the element at position p: stored by id, or already in the order
// of the positions (in_order: a previous pass wrote them permuted).
__device__ __forceinline__ int32_t elem_key(const int32_t* keys, const int32_t* in_ids,
                                            int64_t p, bool in_order) {
  return in_order ? keys[p] : keys[elem_id(in_ids, p)];
}

template <bool kMulti>
__global__ void __launch_bounds__(kSortThreads) k_sort_hist(const __grid_constant__ SortBatch b) {
  const SortSeg& g = b.seg[kMulti ? blockIdx.y : 0];
  if (int64_t(blockIdx.x) >= g.tiles) return;
  extern __shared__ int32_t sh_cnt[];
  const int digits = 1 << b.bits, mask = digits - 1, shift = b.shift;
  for (int i = threadIdx.x; i < digits; i += blockDim.x) sh_cnt[i] = 0;
  __syncthreads();
  const int64_t base = int64_t(blockIdx.x) * kSortTile;
  // an element counts when it lies inside the segment (p < M), whatever its key: the
  // scatter ranks exactly those elements by the same digit expression, so a key outside
  // [0, 2^bits) -- a negative one included -- is sorted by its low bits on both sides
  int32_t kv[kSortTile / kSortThreads];
#pragma unroll
  for (int u = 0; u < kSortTile / kSortThreads; ++u) {
    const int64_t p = base + u * kSortThreads + threadIdx.x;
    kv[u] = p < g.M ? elem_key(g.keys, g.in_ids, p, b.in_order) : 0;
  }
#pragma unroll
  for (int u = 0; u < kSortTile / kSortThreads; ++u)
    if (base + u * kSortThreads + threadIdx.x < g.M)
      atomicAdd(&sh_cnt[(kv[u] >> shift) & mask], 1);
  __syncthreads();
  for (int i = threadIdx.x; i < digits; i += blockDim.x)
    g.hist[int64_t(i) * g.tiles + blockIdx.x] = sh_cnt[i];
}

// Exclusive block scan of one value per thread; returns the exclusive prefix and
// writes the block total to *total (all threads see it after the call).
__device__ int32_t block_exclusive_scan(int32_t v, int32_t* sh_warp, int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) sh_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t w = lane < nw ? sh_warp[lane] : 0;
    int32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t u = __shfl_up_sync(0xFFFFFFFFu, wi, o);
      if (lane >= o) wi += u;
    }
    if (lane < nw) sh_warp[lane] = wi - w;
    if (lane == nw - 1) *total = wi;
  }
  __syncthreads();
  const int32_t r = sh_warp[warp] + incl - v;
  __syncthreads();
  return r;
}

// grid = (digits, segments); row d of hist becomes its exclusive prefix over tiles; the
// total goes to start[d].
template <bool kMulti>
__global__ void __launch_bounds__(256) k_sort_scan_tiles(const __grid_constant__ SortBatch b) {
  const SortSeg& g = b.seg[kMulti ? blockIdx.y : 0];
  __shared__ int32_t sh_warp[32];
  __shared__ int32_t sh_total;
  int32_t* row = g.hist + int64_t(blockIdx.x) * g.tiles;
  int32_t carry = 0;
  for (int64_t c0 = 0; c0 < g.tiles; c0 += blockDim.x) {
    const int64_t i = c0 + threadIdx.x;
    const int32_t v = i < g.tiles ? row[i] : 0;
    const int32_t ex = block_exclusive_scan(v, sh_warp, &sh_total);
    if (i < g.tiles) row[i] = carry + ex;
    carry += sh_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) g.start[blockIdx.x] = carry;
}

// One block per segment: start[0..digits) = exclusive prefix of the totals held there;
// start[digits] = M.
template <bool kMulti>
__global__ void __launch_bounds__(1024) k_sort_scan_digits(const __grid_constant__ SortBatch b) {
  const SortSeg& g = b.seg[kMulti ? blockIdx.y : 0];
  const int digits = 1 << b.bits;
  __shared__ int32_t sh_warp[32];
  __shared__ int32_t sh_total;
  int32_t carry = 0;
  for (int c0 = 0; c0 < digits; c0 += blockDim.x) {
    const int i = c0 + threadIdx.x;
    const int32_t v = i < digits ? g.start[i] : 0;
    const int32_t ex = block_exclusive_scan(v, sh_warp, &sh_total);
    if (i < digits) g.start[i] = carry + ex;
    carry += sh_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) g.start[digits] = carry;
}

// Shared memory of the scatter: per-warp digit counts, per-digit offsets, and the tile
// staged in digit order (id, key, payload) so that the global writes are contiguous runs.
__host__ __device__ constexpr size_t scatter_smem_bytes(int bits) {
  return ((size_t(kWarps) * (size_t(1) << bits) * 2 + 15) & ~size_t(15))  // cnt (uint16)
         + size_t(3) * 4 * (size_t(1) << bits)                            // offsets
         + size_t(kSortTile) * 12;                                        // staged tile
}

template <bool kMulti>
__global__ void __launch_bounds__(kSortThreads, 4) k_sort_scatter(const __grid_constant__ SortBatch b) {
  const SortSeg& g = b.seg[kMulti ? blockIdx.y : 0];
  if (int64_t(blockIdx.x) >= g.tiles) return;
  const int32_t* __restrict__ keys = g.keys;
  const int32_t* __restrict__ in_ids = g.in_ids;
  const int64_t M = g.M, tiles = g.tiles;
  const int shift = b.shift;
  const bool in_order = b.in_order;
  const int32_t* __restrict__ hist = g.hist;
  const int32_t* __restrict__ digit_start = g.start;
  int32_t* __restrict__ out_ids = g.out_ids;
  int32_t* __restrict__ out_keys = g.out_keys;
  const float* __restrict__ payload = g.payload;
  float* __restrict__ out_payload = g.out_payload;
  extern __shared__ __align__(16) unsigned char sh_raw[];
  const int digits = 1 << b.bits, mask = digits - 1;
  uint16_t* cnt = reinterpret_cast<uint16_t*>(sh_raw);  // [kWarps][digits]
  int32_t* gbase = reinterpret_cast<int32_t*>(sh_raw + ((kWarps * digits * 2 + 15) & ~15));
  int32_t* lbase = gbase + digits;   // first staged position of each digit in this tile
  int32_t* total = lbase + digits;   // this tile's count of each digit
  int32_t* s_id = total + digits;
  int32_t* s_key = s_id + kSortTile;
  float* s_pay = reinterpret_cast<float*>(s_key + kSortTile);
  __shared__ int32_t sh_warp[32];
  __shared__ int32_t sh_total;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t tile = blockIdx.x;
  const int64_t tile0 = tile * kSortTile;
  const int n_tile = int(M - tile0 < kSortTile ? M - tile0 : kSortTile);

  for (int i = tid; i < kWarps * digits; i += blockDim.x) cnt[i] = 0;
  for (int i = tid; i < digits; i += blockDim.x)
    gbase[i] = digit_start[i] + hist[int64_t(i) * tiles + tile];
  __syncthreads();

  const int64_t wbase = tile0 + int64_t(warp) * kPerWarp;
  uint16_t* wcnt = cnt + warp * digits;
  // every lane's 16 elements (one per warp step), loaded up front, all in flight together
  int32_t r_id[kSteps], r_key[kSteps];
  float r_pay[kSteps];
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const int64_t p = wbase + s * 32 + lane;
    r_id[s] = 0;
    r_key[s] = 0;
    r_pay[s] = 0.0f;
    if (p < M) {
      r_id[s] = elem_id(in_ids, p);
      r_key[s] = in_order ? keys[p] : keys[r_id[s]];
      if (payload) r_pay[s] = in_order ? payload[p] : payload[r_id[s]];
    }
  }
  // pass 1: this warp's count of every digit
  unsigned r_peers[kSteps];
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const bool ok = wbase + s * 32 + lane < M;
    const int dg = (r_key[s] >> shift) & mask;
    const unsigned peers = digit_peers(dg, b.bits, ok, lane);
    r_peers[s] = peers;
    if (ok && lane == __ffs(peers) - 1) wcnt[dg] += uint16_t(__popc(peers));
    __syncwarp();
  }
  __syncthreads();
  // per digit: exclusive prefix over the warps; the tile's total
  for (int dg = tid; dg < digits; dg += blockDim.x) {
    uint16_t run = 0;
    for (int w = 0; w < kWarps; ++w) {
      const uint16_t c = cnt[w * digits + dg];
      cnt[w * digits + dg] = run;
      run = uint16_t(run + c);
    }
    total[dg] = run;
  }
  __syncthreads();
  // staged position of each digit's first element: exclusive scan of the totals
  int32_t carry = 0;
  for (int c0 = 0; c0 < digits; c0 += blockDim.x) {
    const int dg = c0 + tid;
    const int32_t v = dg < digits ? total[dg] : 0;
    const int32_t ex = block_exclusive_scan(v, sh_warp, &sh_total);
    if (dg < digits) lbase[dg] = carry + ex;
    carry += sh_total;
    __syncthreads();
  }
  // pass 2: stage every element at its rank, in order
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const bool ok = wbase + s * 32 + lane < M;
    const int32_t key = r_key[s];
    const int dg = (key >> shift) & mask;
    const unsigned peers = r_peers[s];
    const int base = ok ? int(wcnt[dg]) : 0;
    __syncwarp();
    if (ok) {
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int lp = lbase[dg] + base + rank;
      s_id[lp] = r_id[s];
      s_key[lp] = key;
      s_pay[lp] = r_pay[s];
      if (lane == __ffs(peers) - 1) wcnt[dg] = uint16_t(base + __popc(peers));
    }
    __syncwarp();
  }
  __syncthreads();
  // write out: consecutive staged positions of a digit go to consecutive global positions
  for (int lp = tid; lp < n_tile; lp += blockDim.x) {
    const int32_t key = s_key[lp];
    const int dg = (key >> shift) & mask;
    const int64_t pos = int64_t(gbase[dg]) + (lp - lbase[dg]);
    out_ids[pos] = s_id[lp];
    if (out_keys) out_keys[pos] = key;
    if (out_payload) out_payload[pos] = s_pay[lp];
  }
}

// start[j] = first position p of sorted (non-decreasing) keys with key >= j, j in [0, n_vals]:
// one thread per value, a binary search.  (Filling the gap below each key from the key's
// own thread left one thread to write every value above the largest key, millions of them
// when the keys are few and crowd the low values, as a batch's Zipf-drawn targets do.)
__global__ void __launch_bounds__(256) k_segment_starts(const int32_t* __restrict__ sorted,
                                                        int64_t M, int32_t n_vals,
                                                        int32_t* __restrict__ start) {
  for (int64_t j = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; j <= n_vals;
       j += int64_t(gridDim.x) * blockDim.x) {
    int64_t lo = 0, hi = M;
    while (lo < hi) {
      const int64_t mid = (lo + hi) >> 1;
      if (__ldg(sorted + mid) < j) lo = mid + 1;
      else hi = mid;
    }
    start[j] = int32_t(lo);
  }
}

}  // namespace

cudaError_t launch_segment_starts(const int32_t* sorted, int64_t M, int32_t n_vals,
                                  int32_t* start, cudaStream_t st) {
  const int64_t want = ceil_div(int64_t(n_vals) + 1, 256);
  k_segment_starts<<<unsigned(want < 32 * 148 ? want : 32 * 148), 256, 0, st>>>(sorted, M,
                                                                               n_vals, start);
  count_launches(1);
  return cudaGetLastError();
}

// The single-segment kernels index the segment statically (its fields stay kernel
// parameters); the batch kernels pick it by blockIdx.y.
template <bool kMulti>
cudaError_t run_sort_batch(const SortBatch& b, int64_t max_tiles, int digits, cudaStream_t st) {
  const unsigned n = unsigned(b.n);
  // segments with no element still get their starts (all zero) from the scans
  if (max_tiles > 0)
    k_sort_hist<kMulti><<<dim3(unsigned(max_tiles), n), kSortThreads, sizeof(int32_t) * digits,
                          st>>>(b);
  k_sort_scan_tiles<kMulti><<<dim3(digits, n), 256, 0, st>>>(b);
  k_sort_scan_digits<kMulti><<<dim3(1, n), 1024, 0, st>>>(b);
  count_launches(2);
  if (max_tiles > 0) {
    // Opt in to the largest dynamic shared memory the scatter can use (per device; cheap).
    cudaError_t e = cudaFuncSetAttribute(k_sort_scatter<kMulti>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(scatter_smem_bytes(kMaxDigitBits)));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k_sort_scatter<kMulti>,
                             cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    k_sort_scatter<kMulti><<<dim3(unsigned(max_tiles), n), kSortThreads,
                             scatter_smem_bytes(b.bits), st>>>(b);
    count_launches(2);
  }
  return cudaGetLastError();
}

cudaError_t launch_sort_batch(const SortSeg* segs, int n, int shift, int bits, bool in_order,
                              cudaStream_t st) {
  if (n < 1 || n > kMaxSortSegs) return cudaErrorInvalidValue;
  SortBatch b{};
  int64_t max_tiles = 0;
  for (int i = 0; i < n; ++i) {
    b.seg[i] = segs[i];
    b.seg[i].tiles = ceil_div(segs[i].M, kSortTile);
    if (b.seg[i].tiles > max_tiles) max_tiles = b.seg[i].tiles;
  }
  b.n = n;
  b.shift = shift;
  b.bits = bits;
  b.in_order = in_order;
  const int digits = 1 << bits;
  return n > 1 ? run_sort_batch<true>(b, max_tiles, digits, st)
               : run_sort_batch<false>(b, max_tiles, digits, st);
}

cudaError_t launch_sort_pass(const int32_t* keys, const int32_t* in_ids, int64_t M, int shift,
                             int bits, void* scratch, int32_t* out_ids, int32_t* out_keys,
                             int32_t* digit_start, cudaStream_t st, const float* payload,
                             float* out_payload, bool in_order) {
  const int digits = 1 << bits;
  const int64_t tiles = ceil_div(M > 0 ? M : 1, kSortTile);
  SortSeg g{};
  g.keys = keys;
  g.in_ids = in_ids;
  g.M = M;
  g.hist = static_cast<int32_t*>(scratch);
  g.start = digit_start ? digit_start
                        : reinterpret_cast<int32_t*>(static_cast<char*>(scratch) +
                                                     align256(sizeof(int32_t) * size_t(digits * tiles)));
  g.out_ids = out_ids;
  g.out_keys = out_keys;
  g.payload = payload;
  g.out_payload = out_payload;
  return launch_sort_batch(&g, 1, shift, bits, in_order, st);
}

}  // namespace rece
