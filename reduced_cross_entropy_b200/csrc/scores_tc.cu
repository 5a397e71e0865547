// scores_tc.cu -- steps 3-4 for large d on the tcgen05 tensor cores (bf16 mode): the
// chunk-window scores (RECE, section 3, Algorithm 1: chunk sets, neighbour window, chunk
// logits; the rounds paragraph) computed once, then each row's candidates for its top-k
// negatives (SCE abstract) selected from them.
//
// At large d one 128 x 128 score tile costs 128 x 128 x d multiply-adds, so the fused
// kernel's three passes over recomputed tiles (select_tc.cu) triple the tensor work and
// re-stream both operands from L2 each time.  Here:
//
//   k_scores_tc     work item = (round r, 128 sorted rows, group of 4 column tiles of the
//                   union of their windows).  K-outer: every 64-wide slab of d brings the
//                   rows' slab of Xs once and the 4 tiles' slabs of Ys (TMA, 128-byte
//                   swizzle) and one thread issues the 4 MMAs into 4 TMEM accumulators of
//                   128 x 128 fp32; four epilogue warpgroups (one per accumulator) then
//                   write the scores, fp32, to a buffer S[r][p][column of the union].
//   k_select_scores one warp per (round, sorted row), reading the row's window of S three
//                   times (from L2, mostly): the same exact selection as the fused kernel --
//                   max, histogram of the order-key distance below it (8 bins per binade,
//                   256 bins), the cut bin b* where the cumulative count reaches E = k + 1,
//                   and every score >= the threshold t at the lower edge of b* emitted as
//                   (score, sorted position) into the row's lists, with the largest fp32
//                   value below t as the bound of what was left out.
//
// The lists have the fused kernel's format (four sub-lists of Qw entries, entry e of the
// row in sub-list e mod 4, so their shares are even as the fused kernel's are), so the
// merge and its exactness check are shared.  The scores pass through HBM
// once (4 bytes per window score); that is far cheaper than recomputing d-deep dot
// products at the sizes this path is chosen for.
#include "common.cuh"
#include "plan.h"
#include "sm100.cuh"
#include "tc.h"
#include "tc_bins.cuh"

namespace rece {
namespace {

using namespace sm100;
using namespace tcsel;

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kBK = 64;
constexpr int kGroup = 4;  // column tiles per work item (4 x 128 TMEM columns)
constexpr int kStages = 2;
constexpr uint32_t kSlabA = kBM * kBK * 2;  // 16 KB
constexpr uint32_t kSlabB = kBN * kBK * 2;  // 16 KB per tile
constexpr int kEpiWarps = 4 * kGroup;
constexpr int kThreads = 64 + kEpiWarps * 32;
constexpr uint64_t kTimeoutNs = 1000000000ull;

struct __align__(1024) ScoreSmem {
  uint8_t a[kStages][kSlabA];
  uint8_t b[kStages][kGroup][kSlabB];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ int64_t chunk_of(int64_t p, int64_t M, int n_c) {
  return (p * n_c) / M;
}

struct Item {
  int r;
  int64_t p0;  // first sorted row
  int64_t U0;  // union window start (sorted catalogue position)
  int64_t W;   // union width
  int t0;      // first column tile of the group (within the union)
  int nt;      // tiles of the group (0: nothing to do)
};

// Work item w = ((r * tiles_per_round) + row tile) * groups + g.
__device__ __forceinline__ Item item_of(int64_t w, int64_t tiles_per_round, int groups, int64_t N,
                                        int64_t C, int n_c, int n_ec) {
  Item it;
  const int g = int(w % groups);
  const int64_t rt = w / groups;
  it.r = int(rt / tiles_per_round);
  it.p0 = (rt % tiles_per_round) * kBM;
  const int64_t last = (it.p0 + kBM - 1 < N - 1) ? it.p0 + kBM - 1 : N - 1;
  const int64_t cf = chunk_of(it.p0, N, n_c), cl = chunk_of(last, N, n_c);
  it.U0 = chunk_start(cf - n_ec < 0 ? 0 : cf - n_ec, C, n_c);
  const int64_t U1 = chunk_start(cl + n_ec + 1 > n_c ? n_c : cl + n_ec + 1, C, n_c);
  it.W = U1 - it.U0;
  const int nt_all = int((it.W + kBN - 1) / kBN);
  it.t0 = g * kGroup;
  it.nt = nt_all - it.t0;
  it.nt = it.nt < 0 ? 0 : (it.nt > kGroup ? kGroup : it.nt);
  return it;
}

__device__ __forceinline__ void on_timeout(ScoreSmem& s, uint32_t* status) {
  *reinterpret_cast<volatile int*>(&s.abort) = 1;
  raise_flag(status, RECE_DEVICE_TIMEOUT);
}

__global__ void __launch_bounds__(kThreads, 1) k_scores_tc(
    const __grid_constant__ CUtensorMap tmXs, const __grid_constant__ CUtensorMap tmYs,
    int64_t N, int64_t C, int d, int n_c, int n_ec, int n_r, int groups, int64_t Wp,
    float* __restrict__ S, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  ScoreSmem& s = *reinterpret_cast<ScoreSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tiles_per_round = (N + kBM - 1) / kBM;
  const int64_t items = tiles_per_round * n_r * groups;
  const int nk = d / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(&s.acc_full, 1);
    mbar_init(&s.acc_empty, kEpiWarps);
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
    if (lane == 0) {
      prefetch_tmap(&tmXs);
      prefetch_tmap(&tmYs);
      uint32_t it = 0;
      for (int64_t w = blockIdx.x; w < items && !*abortp; w += gridDim.x) {
        const Item I = item_of(w, tiles_per_round, groups, N, C, n_c, n_ec);
        if (I.nt == 0) continue;
        const int32_t arow = int32_t(int64_t(I.r) * N + I.p0);
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int st = it % kStages;
          if (!mbar_wait(&s.empty[st], ((it / kStages) & 1u) ^ 1u, &s.abort, kTimeoutNs)) {
            on_timeout(s, status);
            break;
          }
          mbar_arrive_expect_tx(&s.full[st], kSlabA + uint32_t(I.nt) * kSlabB);
          tma_load_2d(s.a[st], &tmXs, &s.full[st], ks * kBK, arow);
          for (int t = 0; t < I.nt; ++t)
            tma_load_2d(s.b[st][t], &tmYs, &s.full[st], ks * kBK,
                        int32_t(int64_t(I.r) * C + I.U0 + int64_t(I.t0 + t) * kBN));
        }
      }
      for (uint32_t j = (it > kStages ? it - kStages : 0); j < it; ++j)
        mbar_wait_limit(&s.full[j % kStages], (j / kStages) & 1u, kTimeoutNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, kBN);
      uint32_t it = 0, ni = 0;
      bool ok = true;
      for (int64_t w = blockIdx.x; w < items && ok && !*abortp; w += gridDim.x) {
        const Item I = item_of(w, tiles_per_round, groups, N, C, n_c, n_ec);
        if (I.nt == 0) continue;
        // the epilogue has drained the previous item's accumulators
        if (!mbar_wait(&s.acc_empty, (ni & 1u) ^ 1u, &s.abort, kTimeoutNs)) {
          on_timeout(s, status);
          break;
        }
        tc_fence_after();
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int st = it % kStages;
          if (!mbar_wait(&s.full[st], (it / kStages) & 1u, &s.abort, kTimeoutNs)) {
            on_timeout(s, status);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = desc_k_sw128(smem_u32(s.a[st]));
          for (int t = 0; t < I.nt; ++t) {
            const uint64_t db = desc_k_sw128(smem_u32(s.b[st][t]));
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              mma_bf16(tmem + t * kBN, da + 2 * kk, db + 2 * kk, idesc, (ks | kk) != 0);
          }
          mma_commit(&s.empty[st]);
        }
        if (!ok) break;
        mma_commit(&s.acc_full);
        ++ni;
      }
      mma_commit(&s.drain);
      mbar_wait_limit(&s.drain, 0, kTimeoutNs);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    // warpgroup wg drains accumulator wg (column tile t0 + wg of the item)
    const int wg = (warp - 2) >> 2;
    const int q4 = warp & 3;  // TMEM lane quarter this warp may access
    const int row_local = q4 * 32 + lane;
    uint32_t ni = 0;
    bool ok = true;
    for (int64_t w = blockIdx.x; w < items; w += gridDim.x) {
      const Item I = item_of(w, tiles_per_round, groups, N, C, n_c, n_ec);
      if (I.nt == 0) continue;
      if (!ok || !mbar_wait(&s.acc_full, ni & 1u, &s.abort, kTimeoutNs)) {
        if (ok) on_timeout(s, status);
        ok = false;
        break;
      }
      tc_fence_after();
      if (wg < I.nt) {
        const int64_t p = I.p0 + row_local;
        const int64_t col0 = int64_t(I.t0 + wg) * kBN;
        const int ncol = int(I.W - col0 < kBN ? I.W - col0 : kBN);
        float* dst = S + (int64_t(I.r) * N + p) * Wp + col0;
        const uint32_t taddr = tmem + (uint32_t(q4 * 32) << 16) + uint32_t(wg * kBN);
        for (int c0 = 0; c0 < kBN; c0 += 32) {
          float v[32];
          tmem_load32(taddr + c0, v);
          if (p >= N) continue;
          if (c0 + 32 <= ncol) {
            float4* o = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
            for (int u = 0; u < 8; ++u)
              o[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
          } else {
#pragma unroll
            for (int u = 0; u < 32; ++u)
              if (c0 + u < ncol) dst[c0 + u] = v[u];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.acc_empty);
      ++ni;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// One warp per (round r, sorted row p): the exact selection of the row's candidates from
// its window of S (see the file comment).  hist: 256 bins per warp in shared memory.
constexpr int kSelThreads = 256;
constexpr int kSelBins = 256;

__global__ void __launch_bounds__(kSelThreads) k_select_scores(
    const float* __restrict__ S, int64_t N, int64_t C, int n_c, int n_ec, int n_r, int64_t Wp,
    int Qw, int E, int2* __restrict__ list, int4* __restrict__ list_count,
    float* __restrict__ list_theta) {
  __shared__ uint32_t hist[kSelThreads / 32][kSelBins];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t w = int64_t(blockIdx.x) * (kSelThreads / 32) + wid;
  if (w >= int64_t(n_r) * N) return;  // whole warp leaves together
  const int64_t p = w % N;
  // the row's window and the union of its 128-row tile (S's columns)
  const int64_t p0 = (p / kBM) * kBM;
  const int64_t cp = chunk_of(p, N, n_c), cf = chunk_of(p0, N, n_c);
  const int64_t U0 = chunk_start(cf - n_ec < 0 ? 0 : cf - n_ec, C, n_c);
  const int64_t w0 = chunk_start(cp - n_ec < 0 ? 0 : cp - n_ec, C, n_c);
  const int64_t w1 = chunk_start(cp + n_ec + 1 > n_c ? n_c : cp + n_ec + 1, C, n_c);
  const int W = int(w1 - w0);
  const float* sc = S + w * Wp + (w0 - U0);
  uint32_t* h = hist[wid];

  float thr = -INFINITY;  // emit every score >= thr
  if (W > E) {
    float mx = -INFINITY;
    for (int c = lane; c < W; c += 32) mx = fmaxf(mx, sc[c]);
    mx = warp_max(mx);
    for (int b = lane; b < kSelBins; b += 32) h[b] = 0u;
    __syncwarp();
    const BinMap bm = bin_map(mx, 0u);
    for (int c = lane; c < W; c += 32) {
      const uint32_t raw = (__float_as_uint(sc[c]) * bm.sig + bm.off) >> 20;
      if (raw < uint32_t(kSelBins - 1)) atomicAdd(&h[raw], 1u);  // the last bin is open
    }
    __syncwarp();
    // the smallest bin whose cumulative count reaches E: lane l scans bins 8l..8l+7
    uint32_t c8[8], s8 = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      c8[u] = (8 * lane + u < kSelBins - 1) ? h[8 * lane + u] : 0u;
      s8 += c8[u];
    }
    uint32_t incl = s8;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - s8;
    int bstar = 1 << 30;
    if (excl < uint32_t(E) && uint32_t(E) <= incl) {
      uint32_t run = excl;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        run += c8[u];
        if (run >= uint32_t(E)) {
          bstar = 8 * lane + u;
          break;
        }
      }
    }
    int bmin = bstar;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const int v = __shfl_xor_sync(0xFFFFFFFFu, bmin, o);
      bmin = v < bmin ? v : bmin;
    }
    if (bmin < kSelBins - 1) thr = cut_threshold(bm, uint32_t(bmin + 1) << 20);
  }
  // emission, in column order: entry e goes to sub-list e mod 4, slot e / 4
  int2* out = list + w * 4 * int64_t(Qw);
  int n = 0;
  for (int c0 = 0; c0 < W; c0 += 32) {
    const int c = c0 + lane;
    const float v = c < W ? sc[c] : -INFINITY;
    const bool e = c < W && v >= thr;
    const unsigned b = __ballot_sync(0xFFFFFFFFu, e);
    if (e) {
      const int idx = n + __popc(b & ((1u << lane) - 1u));
      if ((idx >> 2) < Qw)
        out[(idx & 3) * Qw + (idx >> 2)] = make_int2(__float_as_int(v), int32_t(w0 + c));
    }
    n += __popc(b);
  }
  if (lane == 0) {
    // entries per sub-list (more than Qw: the list overflowed)
    list_count[w] = make_int4((n + 3) >> 2, (n + 2) >> 2, (n + 1) >> 2, n >> 2);
    list_theta[w] = thr == -INFINITY ? -INFINITY : value_below(thr);
  }
}

}  // namespace

int tc_sublist_capacity(int k);
int tc_emit_target(int k);

// Longest union of windows over the 128-row tiles (the columns of S per row).
int64_t scores_tc_width(const rece_plan_s& p) {
  const auto& c = p.cfg;
  int64_t wmax = 0;
  for (int64_t p0 = 0; p0 < c.N; p0 += kBM) {
    const int64_t last = (p0 + kBM - 1 < c.N - 1) ? p0 + kBM - 1 : c.N - 1;
    const int64_t cf = (p0 * c.n_c) / c.N, cl = (last * c.n_c) / c.N;
    const int64_t U0 = chunk_start(cf - c.n_ec < 0 ? 0 : cf - c.n_ec, c.C, c.n_c);
    const int64_t U1 = chunk_start(cl + c.n_ec + 1 > c.n_c ? c.n_c : cl + c.n_ec + 1, c.C, c.n_c);
    if (U1 - U0 > wmax) wmax = U1 - U0;
  }
  return (wmax + 3) / 4 * 4;
}

cudaError_t launch_scores_select_tc(const rece_plan_s& p, const void* Xs, const void* Ys,
                                    float* S, int2* list, int4* list_count, float* list_theta,
                                    uint32_t* status, cudaStream_t st) {
  const auto& c = p.cfg;
  if (c.N == 0) return cudaSuccess;
  CUtensorMap tmXs, tmYs;
  cudaError_t e = make_tmap_bf16(&tmXs, Xs, uint64_t(c.n_r) * c.N, c.d, kBM);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tmYs, Ys, uint64_t(c.n_r) * c.C, c.d, kBN);
  if (e != cudaSuccess) return e;
  const int64_t Wp = p.score_width;
  const int groups = int((Wp + kGroup * kBN - 1) / (kGroup * kBN));
  const int64_t items = ceil_div(c.N, kBM) * c.n_r * groups;
  const int grid = int(items < sm_count() ? items : sm_count());
  const size_t smem = sizeof(ScoreSmem) + 1024;
  e = cudaFuncSetAttribute(k_scores_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  k_scores_tc<<<grid, kThreads, smem, st>>>(tmXs, tmYs, c.N, c.C, c.d, c.n_c, c.n_ec, c.n_r,
                                            groups, Wp, S, status);
  const int64_t rows = int64_t(c.n_r) * c.N;
  k_select_scores<<<unsigned(ceil_div(rows, kSelThreads / 32)), kSelThreads, 0, st>>>(
      S, c.N, c.C, c.n_c, c.n_ec, c.n_r, Wp, tc_sublist_capacity(c.k), tc_emit_target(c.k),
      list, list_count, list_theta);
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace rece
