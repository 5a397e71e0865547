// bucketize_tc.cu -- step 1 on the tcgen05 tensor cores (bf16 mode): for every row v of
// X and of Y and every round r, bucket = argmax_b <B[r][b], v> (RECE, section 3,
// Algorithm 1, the argmax steps); ties go to the lowest b.
//
// A persistent, warp-specialised GEMM with the argmax fused into its epilogue:
//   warp 0      TMA producer: per stage one 128-row x 64 slice of V and one up-to-256-row
//               x 64 slice of B_r (128-byte swizzle), 4 stages in flight;
//   warp 1      MMA issuer: M=128 x N=bn x K=16 tcgen05.mma per 32-byte step, fp32
//               accumulators in TMEM, two 256-column buffers so the epilogue of one tile
//               overlaps the MMAs of the next;
//   warps 2-5   epilogue: thread = row; reads its row of the accumulator with
//               tcgen05.ld and keeps the running (max, argmax).
// The (rows x n_b) projection matrix never leaves the chip.  Work item = (round, 128-row
// tile of X or Y); the CTA loops over items with a grid stride.
#include <climits>

#include "common.cuh"
#include "plan.h"
#include "sm100.cuh"
#include "tc.h"

namespace rece {
namespace {

using namespace sm100;

constexpr int kStages = 4;
constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr uint32_t kStageABytes = kBM * kBK * 2;  // 16 KB
constexpr uint32_t kStageBBytes = kBN * kBK * 2;  // 32 KB
constexpr uint64_t kTimeoutNs = 1000000000ull;    // 1 s per wait
constexpr int kThreads = 192;

struct __align__(1024) Smem {
  uint8_t a[kStages][kStageABytes];
  uint8_t b[kStages][kStageBBytes];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Running (max, argmax) over the scores v[0..32) of vectors b0..b0+31 (those >= n_b
// excluded), ties to the lowest b: the earlier chunk keeps a tie (strict >), and inside a
// chunk the first u whose score equals the chunk's maximum wins.  A full chunk costs a
// max tree (one instruction a score); the index is searched only when the chunk beats
// the running best, which gets rare as the best rises.  NaN scores never win.
__device__ __forceinline__ void argmax32(const float (&v)[32], int b0, int n_b, float& best,
                                         int& best_b) {
  if (b0 + 32 <= n_b) {
    float m[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) m[u] = fmaxf(v[2 * u], v[2 * u + 1]);
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
      for (int u = 0; u < w; ++u) m[u] = fmaxf(m[u], m[u + w]);
    if (m[0] > best) {
      int idx = 31;
#pragma unroll
      for (int u = 31; u >= 0; --u)
        if (v[u] == m[0]) idx = u;
      best = m[0];
      best_b = b0 + idx;
    }
  } else {
#pragma unroll
    for (int u = 0; u < 32; ++u)
      if (b0 + u < n_b && v[u] > best) {
        best = v[u];
        best_b = b0 + u;
      }
  }
}

__device__ __forceinline__ void on_timeout(Smem& s, uint32_t* status) {
  *reinterpret_cast<volatile int*>(&s.abort) = 1;
  raise_flag(status, RECE_DEVICE_TIMEOUT);
}

__global__ void __launch_bounds__(kThreads, 1) k_bucketize_tc(
    const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
    const __grid_constant__ CUtensorMap tmB, int64_t N, int64_t C, int d, int n_b, int n_r,
    int bn, int32_t* __restrict__ bx, int32_t* __restrict__ by, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tX = (N + kBM - 1) / kBM, tY = (C + kBM - 1) / kBM;
  const int64_t per_round = tX + tY, items = per_round * n_r;
  const int n_nt = (n_b + kBN - 1) / kBN;
  const int nk = d / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.acc_full[i], 1);
      mbar_init(&s.acc_empty[i], 4);
    }
    mbar_init(&s.drain, 1);
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  volatile int* abortp = &s.abort;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    uint32_t it = 0;
    if (lane == 0) {
      prefetch_tmap(&tmX);
      prefetch_tmap(&tmY);
      prefetch_tmap(&tmB);
      for (int64_t item = blockIdx.x; item < items && !*abortp; item += gridDim.x) {
        const int r = int(item / per_round);
        const int64_t t = item % per_round;
        const bool isY = t >= tX;
        const int64_t row0 = (isY ? t - tX : t) * kBM;
        for (int nt = 0; nt < n_nt && !*abortp; ++nt) {
          for (int ks = 0; ks < nk; ++ks, ++it) {
            const int st = it % kStages;
            const uint32_t n = it / kStages;
            if (!mbar_wait(&s.empty[st], (n & 1u) ^ 1u, &s.abort, kTimeoutNs)) {
              on_timeout(s, status);
              break;
            }
            mbar_arrive_expect_tx(&s.full[st], kStageABytes + uint32_t(bn) * kBK * 2);
            tma_load_2d(s.a[st], isY ? &tmY : &tmX, &s.full[st], ks * kBK, int32_t(row0));
            tma_load_2d(s.b[st], &tmB, &s.full[st], ks * kBK, r * n_b + nt * kBN);
          }
        }
      }
      // teardown: the last load of every stage has landed (or we give up after the limit)
      for (uint32_t j = (it > kStages ? it - kStages : 0); j < it; ++j)
        mbar_wait_limit(&s.full[j % kStages], (j / kStages) & 1u, kTimeoutNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, bn);
      uint32_t it = 0, acc_it = 0;
      for (int64_t item = blockIdx.x; item < items && !*abortp; item += gridDim.x) {
        for (int nt = 0; nt < n_nt && !*abortp; ++nt, ++acc_it) {
          const int a = acc_it & 1;
          const uint32_t m = acc_it >> 1;
          if (!mbar_wait(&s.acc_empty[a], (m & 1u) ^ 1u, &s.abort, kTimeoutNs)) {
            on_timeout(s, status);
            break;
          }
          tc_fence_after();
          bool ok = true;
          for (int ks = 0; ks < nk; ++ks, ++it) {
            const int st = it % kStages;
            if (!mbar_wait(&s.full[st], (it / kStages) & 1u, &s.abort, kTimeoutNs)) {
              on_timeout(s, status);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t da = desc_k_sw128(smem_u32(s.a[st]));
            const uint64_t db = desc_k_sw128(smem_u32(s.b[st]));
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              mma_bf16(tmem + a * kBN, da + 2 * kk, db + 2 * kk, idesc, (ks | kk) != 0);
            mma_commit(&s.empty[st]);
          }
          if (!ok) break;
          mma_commit(&s.acc_full[a]);
        }
      }
      // teardown: every MMA issued so far has completed
      mma_commit(&s.drain);
      mbar_wait_limit(&s.drain, 0, kTimeoutNs);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row_local = q * 32 + lane;
    uint32_t acc_it = 0;
    for (int64_t item = blockIdx.x; item < items && !*abortp; item += gridDim.x) {
      const int r = int(item / per_round);
      const int64_t t = item % per_round;
      const bool isY = t >= tX;
      const int64_t row0 = (isY ? t - tX : t) * kBM;
      float best = -INFINITY;
      int best_b = INT_MAX;
      bool ok = true;
      for (int nt = 0; nt < n_nt; ++nt, ++acc_it) {
        const int a = acc_it & 1;
        if (!mbar_wait(&s.acc_full[a], (acc_it >> 1) & 1u, &s.abort, kTimeoutNs)) {
          on_timeout(s, status);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem + (uint32_t(q * 32) << 16) + uint32_t(a * kBN);
        for (int c0 = 0; c0 < bn; c0 += 32) {
          float v[32];
          tmem_load32(taddr + c0, v);
          argmax32(v, nt * kBN + c0, n_b, best, best_b);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.acc_empty[a]);
      }
      if (!ok) break;
      const int64_t row = row0 + row_local;
      const int64_t M = isY ? C : N;
      if (row < M) (isY ? by : bx)[int64_t(r) * M + row] = best_b;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The same for d <= 256, with the rows kept resident: work item = (round, 256-row tile of
// X or Y) whose two 128-row blocks (all of d: at most 4 slices of 64) are loaded once,
// while only B_r streams, in 128-vector x 64 slices.  Each B slice feeds both row blocks
// (two MMAs of M = 128, N = 128), so a B element is read once per 256 rows and an input
// row once per round: three times fewer L2 bytes per multiply-add than the streamed
// kernel, whose (128 + 256)-element slices fed one 128 x 256 tile.  TMEM: one
// accumulator of 128 columns per (row block, buffer).  Eight epilogue warps, a row each.
constexpr int kRBStages = 4;
constexpr int kRBN = 128;                                  // B vectors per slice
constexpr int kRMaxK = 4;                                  // d <= 256
constexpr uint32_t kRSliceA = kBM * kBK * 2;               // 16 KB
constexpr uint32_t kRSliceB = kRBN * kBK * 2;              // 16 KB
constexpr int kRThreads = 64 + 256;

struct __align__(1024) SmemRes {
  uint8_t a[2][kRMaxK][kRSliceA];  // [row block][k slice]
  uint8_t b[kRBStages][kRSliceB];
  uint64_t full[kRBStages];
  uint64_t empty[kRBStages];
  uint64_t a_full, a_empty;
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void on_timeout_res(SmemRes& s, uint32_t* status) {
  *reinterpret_cast<volatile int*>(&s.abort) = 1;
  raise_flag(status, RECE_DEVICE_TIMEOUT);
}

__global__ void __launch_bounds__(kRThreads, 1) k_bucketize_tc_res(
    const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
    const __grid_constant__ CUtensorMap tmB, int64_t N, int64_t C, int d, int n_b, int n_r,
    int bn, int32_t* __restrict__ bx, int32_t* __restrict__ by, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  SmemRes& s = *reinterpret_cast<SmemRes*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kRows = 2 * kBM;
  const int64_t tX = (N + kRows - 1) / kRows, tY = (C + kRows - 1) / kRows;
  const int64_t per_round = tX + tY, items = per_round * n_r;
  const int n_nt = (n_b + kRBN - 1) / kRBN;
  const int nk = d / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRBStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(&s.a_full, 1);
    mbar_init(&s.a_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.acc_full[i], 1);
      mbar_init(&s.acc_empty[i], 8);
    }
    mbar_init(&s.drain, 1);
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  volatile int* abortp = &s.abort;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    uint32_t it = 0, ni = 0;
    bool ok = true;
    if (lane == 0) {
      prefetch_tmap(&tmX);
      prefetch_tmap(&tmY);
      prefetch_tmap(&tmB);
      for (int64_t item = blockIdx.x; item < items && ok && !*abortp;
           item += gridDim.x, ++ni) {
        const int r = int(item / per_round);
        const int64_t t = item % per_round;
        const bool isY = t >= tX;
        const int64_t row0 = (isY ? t - tX : t) * kRows;
        // the rows, once the previous item's MMAs are done with them
        if (!mbar_wait(&s.a_empty, (ni & 1u) ^ 1u, &s.abort, kTimeoutNs)) {
          on_timeout_res(s, status);
          break;
        }
        mbar_arrive_expect_tx(&s.a_full, 2u * uint32_t(nk) * kRSliceA);
        for (int rb = 0; rb < 2; ++rb)
          for (int ks = 0; ks < nk; ++ks)
            tma_load_2d(s.a[rb][ks], isY ? &tmY : &tmX, &s.a_full, ks * kBK,
                        int32_t(row0 + rb * kBM));
        for (int nt = 0; nt < n_nt && ok; ++nt) {
          for (int ks = 0; ks < nk; ++ks, ++it) {
            const int st = it % kRBStages;
            if (!mbar_wait(&s.empty[st], ((it / kRBStages) & 1u) ^ 1u, &s.abort, kTimeoutNs)) {
              on_timeout_res(s, status);
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&s.full[st], uint32_t(bn) * kBK * 2);
            tma_load_2d(s.b[st], &tmB, &s.full[st], ks * kBK, r * n_b + nt * kRBN);
          }
        }
      }
      // teardown: the last loads have landed (or we give up after the limit)
      for (uint32_t j = (it > kRBStages ? it - kRBStages : 0); j < it; ++j)
        mbar_wait_limit(&s.full[j % kRBStages], (j / kRBStages) & 1u, kTimeoutNs);
      if (ni > 0) mbar_wait_limit(&s.a_full, (ni - 1) & 1u, kTimeoutNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, bn);
      uint32_t it = 0, acc_it = 0, ni = 0;
      bool ok = true;
      for (int64_t item = blockIdx.x; item < items && ok && !*abortp;
           item += gridDim.x, ++ni) {
        if (!mbar_wait(&s.a_full, ni & 1u, &s.abort, kTimeoutNs)) {
          on_timeout_res(s, status);
          break;
        }
        for (int nt = 0; nt < n_nt && ok; ++nt, ++acc_it) {
          const int a = acc_it & 1;
          if (!mbar_wait(&s.acc_empty[a], ((acc_it >> 1) & 1u) ^ 1u, &s.abort, kTimeoutNs)) {
            on_timeout_res(s, status);
            ok = false;
            break;
          }
          tc_fence_after();
          for (int ks = 0; ks < nk; ++ks, ++it) {
            const int st = it % kRBStages;
            if (!mbar_wait(&s.full[st], (it / kRBStages) & 1u, &s.abort, kTimeoutNs)) {
              on_timeout_res(s, status);
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t db = desc_k_sw128(smem_u32(s.b[st]));
#pragma unroll
            for (int rb = 0; rb < 2; ++rb) {
              const uint64_t da = desc_k_sw128(smem_u32(s.a[rb][ks]));
#pragma unroll
              for (int kk = 0; kk < kBK / 16; ++kk)
                mma_bf16(tmem + uint32_t(rb * 256 + a * kRBN), da + 2 * kk, db + 2 * kk, idesc,
                         (ks | kk) != 0);
            }
            mma_commit(&s.empty[st]);
          }
          if (!ok) break;
          mma_commit(&s.acc_full[a]);
        }
        if (!ok) break;
        mma_commit(&s.a_empty);  // the rows may be replaced
      }
      // teardown: every MMA issued so far has completed
      mma_commit(&s.drain);
      mbar_wait_limit(&s.drain, 0, kTimeoutNs);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int rb = (warp - 2) >> 2;  // and its row block
    const int row_local = rb * kBM + q * 32 + lane;
    uint32_t acc_it = 0;
    for (int64_t item = blockIdx.x; item < items && !*abortp; item += gridDim.x) {
      const int r = int(item / per_round);
      const int64_t t = item % per_round;
      const bool isY = t >= tX;
      const int64_t row0 = (isY ? t - tX : t) * kRows;
      float best = -INFINITY;
      int best_b = INT_MAX;
      bool ok = true;
      for (int nt = 0; nt < n_nt; ++nt, ++acc_it) {
        const int a = acc_it & 1;
        if (!mbar_wait(&s.acc_full[a], (acc_it >> 1) & 1u, &s.abort, kTimeoutNs)) {
          on_timeout_res(s, status);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr =
            tmem + (uint32_t(q * 32) << 16) + uint32_t(rb * 256 + a * kRBN);
        for (int c0 = 0; c0 < bn; c0 += 32) {
          float v[32];
          tmem_load32(taddr + c0, v);
          argmax32(v, nt * kRBN + c0, n_b, best, best_b);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.acc_empty[a]);
      }
      if (!ok) break;
      const int64_t row = row0 + row_local;
      const int64_t M = isY ? C : N;
      if (row < M) (isY ? by : bx)[int64_t(r) * M + row] = best_b;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


// The same for d <= 256 on pairs of SMs (a cluster of two CTAs, tcgen05 cta_group::2):
// work item = (round, 256-row tile), CTA r of the pair holding rows [128r, 128r + 128) of
// it resident (all of d) and, of every slice of 256 vectors, vectors [128r, 128r + 128)
// (64 K elements a stage); the even CTA issues M = 256 x N = 256 MMAs, each CTA's TMEM
// receiving its own 128 rows (two 256-column accumulators).  An MMA then reads from each
// SM's shared memory half the bytes the single-SM kernel's M = 128 x N = 128 MMAs read
// for the same work (about 120 bytes a clock there, near the SM's 128, which held that
// kernel near 72% of the tensor peak); the rows of the next item load into a second
// buffer meanwhile.  Loads of
// both CTAs complete on the even CTA's barriers; the MMA commits (a stage or a row buffer
// free, an accumulator full, all done) arrive on both CTAs' barriers at once (forwarding
// them from the even CTA's threads instead made the kernel 1.6 times slower).  Eight
// epilogue warps a CTA (warps 3-10): epilogue warps e and e + 4 share the TMEM lanes of
// their warp number mod 4 and take the two column halves of a slice, combined at the end
// of the item (ties to the lower vector).
constexpr int kPStages = 6;
constexpr int kPBN = 256;                        // vectors per slice (N of the pair MMA)
constexpr uint32_t kPSliceA = kBM * kBK * 2;     // 16 KB: 128 rows x 64 K
constexpr uint32_t kPSliceB = 128 * kBK * 2;     // 16 KB: this CTA's 128 vectors x 64 K
constexpr int kPThreads = 96 + 256;              // B loads, MMA, row loads, 8 epilogue warps

struct __align__(1024) SmemPair {
  uint8_t a[2][kRMaxK][kPSliceA];  // [row buffer][k slice]
  uint8_t b[kPStages][kPSliceB];
  uint64_t full[kPStages];
  uint64_t empty[kPStages];
  uint64_t a_full[2], a_empty[2];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  float cmb_v[kBM];
  int cmb_i[kBM];
};
static_assert(sizeof(SmemPair) + 1024 <= 232448, "pair kernel shared memory");

__device__ __forceinline__ void on_timeout_pair(SmemPair& s, uint32_t* status) {
  *reinterpret_cast<volatile int*>(&s.abort) = 1;
  raise_flag(status, RECE_DEVICE_TIMEOUT);
}

__global__ void __launch_bounds__(kPThreads, 1) k_bucketize_tc_pair(
    const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
    const __grid_constant__ CUtensorMap tmB, int64_t N, int64_t C, int d, int n_b, int n_r,
    int32_t* __restrict__ bx, int32_t* __restrict__ by, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  SmemPair& s = *reinterpret_cast<SmemPair*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool lead = rank == 0;
  constexpr int kRows = 2 * kBM;
  const int64_t tX = (N + kRows - 1) / kRows, tY = (C + kRows - 1) / kRows;
  const int64_t per_round = tX + tY, items = per_round * n_r;
  const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int n_nt = (n_b + kPBN - 1) / kPBN;
  const int nk = d / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.a_full[i], 1);
      mbar_init(&s.a_empty[i], 1);
      mbar_init(&s.acc_full[i], 1);
      mbar_init(&s.acc_empty[i], 16);  // the pair's 16 epilogue warps (even CTA's)
    }
    mbar_init(&s.drain, 1);
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&s.tmem_base, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers and TMEM ready before either touches the other
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  volatile int* abortp = &s.abort;

  if (warp == 0) {
    // ---------------------------------------------------------------- B loads
    uint32_t it = 0;
    if (lane == 0) {
      prefetch_tmap(&tmB);
      bool ok = true;
      for (int64_t item = pair; item < items && ok && !*abortp; item += npairs) {
        const int r = int(item / per_round);
        for (int nt = 0; nt < n_nt && ok; ++nt) {
          for (int ks = 0; ks < nk; ++ks, ++it) {
            const int st = it % kPStages;
            if (!mbar_wait_cluster(&s.empty[st], ((it / kPStages) & 1u) ^ 1u, &s.abort,
                                   kTimeoutNs)) {
              on_timeout_pair(s, status);
              ok = false;
              break;
            }
            if (lead) mbar_arrive_expect_tx(&s.full[st], 2 * kPSliceB);  // both halves
            tma_load_2d_pair(s.b[st], &tmB, &s.full[st], ks * kBK,
                             r * n_b + nt * kPBN + int(rank) * 128);
          }
        }
      }
      if (lead)  // teardown: the last stages' loads (both CTAs') have landed
        for (uint32_t j = (it > kPStages ? it - kPStages : 0); j < it; ++j)
          mbar_wait_limit(&s.full[j % kPStages], (j / kPStages) & 1u, kTimeoutNs);
    }
  } else if (warp == 2) {
    // ---------------------------------------------------------------- row loads
    uint32_t ni = 0;
    if (lane == 0) {
      prefetch_tmap(&tmX);
      prefetch_tmap(&tmY);
      for (int64_t item = pair; item < items && !*abortp; item += npairs, ++ni) {
        const int64_t t = item % per_round;
        const bool isY = t >= tX;
        const int64_t row0 = (isY ? t - tX : t) * kRows + int64_t(rank) * kBM;
        const int slot = int(ni & 1u);
        if (!mbar_wait_cluster(&s.a_empty[slot], ((ni >> 1) & 1u) ^ 1u, &s.abort, kTimeoutNs)) {
          on_timeout_pair(s, status);
          break;
        }
        if (lead) mbar_arrive_expect_tx(&s.a_full[slot], 2u * uint32_t(nk) * kPSliceA);
        for (int ks = 0; ks < nk; ++ks)
          tma_load_2d_pair(s.a[slot][ks], isY ? &tmY : &tmX, &s.a_full[slot], ks * kBK,
                           int32_t(row0));
      }
      if (lead)
        for (uint32_t j = (ni > 2 ? ni - 2 : 0); j < ni; ++j)
          mbar_wait_limit(&s.a_full[j & 1u], (j >> 1) & 1u, kTimeoutNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (even CTA)
    if (lane == 0) {
      if (lead) {
        const uint32_t idesc = idesc_bf16_f32(2 * kBM, kPBN);
        uint32_t it = 0, acc_it = 0, ni = 0;
        bool ok = true;
        for (int64_t item = pair; item < items && ok && !*abortp; item += npairs, ++ni) {
          const int slot = int(ni & 1u);
          if (!mbar_wait(&s.a_full[slot], (ni >> 1) & 1u, &s.abort, kTimeoutNs)) {
            on_timeout_pair(s, status);
            break;
          }
          for (int nt = 0; nt < n_nt && ok; ++nt, ++acc_it) {
            const int a = int(acc_it & 1u);
            if (!mbar_wait_cluster(&s.acc_empty[a], ((acc_it >> 1) & 1u) ^ 1u, &s.abort,
                                   kTimeoutNs)) {
              on_timeout_pair(s, status);
              ok = false;
              break;
            }
            tc_fence_after();
            for (int ks = 0; ks < nk; ++ks, ++it) {
              const int st = it % kPStages;
              if (!mbar_wait(&s.full[st], (it / kPStages) & 1u, &s.abort, kTimeoutNs)) {
                on_timeout_pair(s, status);
                ok = false;
                break;
              }
              tc_fence_after();
              const uint64_t da = desc_k_sw128(smem_u32(s.a[slot][ks]));
              const uint64_t db = desc_k_sw128(smem_u32(s.b[st]));
#pragma unroll
              for (int kk = 0; kk < kBK / 16; ++kk)
                mma_bf16_pair(tmem + uint32_t(a * kPBN), da + 2 * kk, db + 2 * kk, idesc,
                              (ks | kk) != 0);
              mma_commit_pair(&s.empty[st]);
            }
            if (!ok) break;
            mma_commit_pair(&s.acc_full[a]);
          }
          if (!ok) break;
          mma_commit_pair(&s.a_empty[slot]);  // the rows may be replaced
        }
        // teardown: every MMA issued so far has completed, in both SMs
        mma_commit_pair(&s.drain);
      }
      const int never = 0;
      mbar_wait_cluster(&s.drain, 0, &never, kTimeoutNs);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - 3;           // 0..7
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int h = ew >> 2;             // column half of the slice
    const int row_local = q * 32 + lane;
    uint32_t acc_it = 0;
    bool ok = true;
    // every epilogue warp walks every item (meeting every named barrier), doing no more
    // waits once one has timed out
    for (int64_t item = pair; item < items; item += npairs) {
      const int r = int(item / per_round);
      const int64_t t = item % per_round;
      const bool isY = t >= tX;
      const int64_t row0 = (isY ? t - tX : t) * kRows + int64_t(rank) * kBM;
      float best = -INFINITY;
      int best_b = INT_MAX;
      for (int nt = 0; nt < n_nt; ++nt, ++acc_it) {
        const int a = int(acc_it & 1u);
        if (ok && (*abortp || !mbar_wait_cluster(&s.acc_full[a], (acc_it >> 1) & 1u, &s.abort,
                                                 kTimeoutNs))) {
          if (!*abortp) on_timeout_pair(s, status);
          ok = false;
        }
        if (!ok) continue;
        tc_fence_after();
        const uint32_t taddr =
            tmem + (uint32_t(q * 32) << 16) + uint32_t(a * kPBN + h * 128);
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 64) {
          float v[64];
          tmem_load64(taddr + c0, v);
          argmax32(*reinterpret_cast<float(*)[32]>(v), nt * kPBN + h * 128 + c0, n_b, best,
                   best_b);
          argmax32(*reinterpret_cast<float(*)[32]>(v + 32), nt * kPBN + h * 128 + c0 + 32, n_b,
                   best, best_b);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(&s.acc_empty[a], 0);
      }
      // the two column halves of the row: the lower vector wins a tie
      if (h == 1) {
        s.cmb_v[row_local] = best;
        s.cmb_i[row_local] = best_b;
      }
      named_barrier(1, 256);
      if (h == 0 && ok) {
        const float v1 = s.cmb_v[row_local];
        const int i1 = s.cmb_i[row_local];
        if (v1 > best || (v1 == best && i1 < best_b)) best_b = i1;
        const int64_t row = row0 + row_local;
        const int64_t M = isY ? C : N;
        if (row < M) (isY ? by : bx)[int64_t(r) * M + row] = best_b;
      }
      named_barrier(1, 256);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the other may still reach its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_bucketize_tc(const rece_plan_s& p, const void* X, const void* Y,
                                const void* B, int32_t* bx, int32_t* by, uint32_t* status,
                                cudaStream_t st) {
  const auto& c = p.cfg;
  const int bn = c.n_b >= kBN ? kBN : ((c.n_b + 15) / 16) * 16;
  CUtensorMap tmX, tmY, tmB;
  cudaError_t e;
  // an empty X still needs a valid descriptor: point it at Y (no X tile is ever loaded)
  e = make_tmap_bf16(&tmX, c.N > 0 ? X : Y, c.N > 0 ? c.N : c.C, c.d, kBM);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tmY, Y, c.C, c.d, kBM);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tmB, B, uint64_t(c.n_r) * c.n_b, c.d, bn);
  if (e != cudaSuccess) return e;
  if (c.d <= kRMaxK * kBK && int64_t(c.n_b) * c.d >= (int64_t(1) << 19) && sm_count() >= 2) {
    // rows resident on pairs of SMs, B streamed once per 256 rows, M = 256 MMAs: where an
    // item holds enough work (n_b d >= 2^19; at n_b = 4096, d = 256: 7.22 -> 6.29 ms) to
    // carry the pair's per-item costs (at n_b = 1024, d = 128 the single-SM kernel is
    // faster: 0.67 against 0.86 ms)
    e = make_tmap_bf16(&tmB, B, uint64_t(c.n_r) * c.n_b, c.d, 128);
    if (e != cudaSuccess) return e;
    const int64_t items = (ceil_div(c.N, 2 * kBM) + ceil_div(c.C, 2 * kBM)) * c.n_r;
    const int64_t pairs = items < sm_count() / 2 ? items : sm_count() / 2;
    const size_t smem = sizeof(SmemPair) + 1024;
    e = cudaFuncSetAttribute(k_bucketize_tc_pair, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(2 * pairs));
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, k_bucketize_tc_pair, tmX, tmY, tmB, c.N, c.C, c.d, c.n_b,
                           c.n_r, bx, by, status);
    count_launches(1);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  if (c.d <= kRMaxK * kBK) {
    // rows resident, B streamed once per 256 rows
    const int bnr = c.n_b >= kRBN ? kRBN : ((c.n_b + 15) / 16) * 16;
    e = make_tmap_bf16(&tmB, B, uint64_t(c.n_r) * c.n_b, c.d, bnr);
    if (e != cudaSuccess) return e;
    const int64_t items = (ceil_div(c.N, 2 * kBM) + ceil_div(c.C, 2 * kBM)) * c.n_r;
    const int grid = int(items < sm_count() ? items : sm_count());
    const size_t smem = sizeof(SmemRes) + 1024;
    e = cudaFuncSetAttribute(k_bucketize_tc_res, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
    if (e != cudaSuccess) return e;
    k_bucketize_tc_res<<<grid, kRThreads, smem, st>>>(tmX, tmY, tmB, c.N, c.C, c.d, c.n_b,
                                                      c.n_r, bnr, bx, by, status);
    count_launches(1);
    return cudaGetLastError();
  }
  const int64_t items = (ceil_div(c.N, kBM) + ceil_div(c.C, kBM)) * c.n_r;
  const int grid = int(items < sm_count() ? items : sm_count());
  const size_t smem = sizeof(Smem) + 1024;
  e = cudaFuncSetAttribute(k_bucketize_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(smem));
  if (e != cudaSuccess) return e;
  k_bucketize_tc<<<grid, kThreads, smem, st>>>(tmX, tmY, tmB, c.N, c.C, c.d, c.n_b, c.n_r, bn,
                                               bx, by, status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace rece
