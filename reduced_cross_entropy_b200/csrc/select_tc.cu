// select_tc.cu -- steps 3-4 on the tcgen05 tensor cores (bf16 mode): chunk-window scores
// (RECE, section 3, Algorithm 1: chunk sets, neighbour window, chunk logits; the rounds
// paragraph) and the candidates for each row's top-k negatives (SCE abstract).
//
// Work item = (round r, 128 consecutive sorted rows).  Their chunks' windows are a
// contiguous range of sorted catalogue rows (the union of the windows), streamed by TMA in
// 128-row tiles; tcgen05.mma forms the 128 x 128 score tile in TMEM.  Each row's thread
// reads its row of the tile and looks only at columns inside its own window.  The window
// is streamed three times, the threshold found without any assumption on the scores'
// distribution:
//   pass 1  per row: max m of a strided quarter of its window's scores (the first 32
//           columns of every tile; all of them when the window is short);
//   pass 2  per row: exact histogram, in shared memory, of the distance key(A) - key(s)
//           >> 20 where key is the order-preserving integer image of an fp32 score and A
//           lies two binades beyond m -- 8 bins per binade of |s| (256 bins, 32 binades,
//           the last one open), so the bins follow the scores' own scale whatever their
//           distribution (heavy-tailed item norms put the k-th score a dozen binades and
//           more below the row's best).
//           The distance is one integer multiply-add on the score's bits;
//   pass 3  the smallest bin b* whose cumulative count reaches E = k + 1 sets the
//           cut, turned into the fp32 threshold t at the lower edge of bin b*: every score
//           >= t is emitted as (score, sorted position) to the row's list (equal scores
//           share a bin, so a tie is never split).  Each thread builds the bit mask of its
//           32 columns that pass and spends work only on the set bits.
// Each of the four epilogue warpgroups (one per 128-column TMEM accumulator, every fourth
// tile) writes its own sub-list of the row, up to k + 32 entries, and its count of all that
// passed.  The largest fp32 value below t bounds every score not emitted and is recorded
// per row (-inf when the whole window was emitted).  The merge kernel keeps the k best;
// the selection is exact whenever no list overflowed and every round's bound is below
// the k-th kept score, which the merge kernel checks row by row.  Without an overflow
// the check always passes: the round with the highest threshold emitted at least
// E = k + 1 entries, at least k of them negatives and none of them a duplicate that an
// earlier round left out (that round's threshold would be higher still), so the k-th
// kept score is >= every round's threshold.  Score tiles never reach HBM.
#include "common.cuh"
#include "plan.h"
#include "sm100.cuh"
#include "tc.h"
#include "tc_bins.cuh"

namespace rece {
namespace {

using namespace sm100;
using namespace tcsel;

constexpr int kStages = 4;
constexpr int kPasses = 3;
constexpr int kBins = 256;                // 8 per binade: 32 binades below the anchor
constexpr int kBinWords = kBins / 2;      // two 16-bit counts per shared word
constexpr int kHeadBins = 16;          // bins above the pass 1 max (2 binades)
constexpr int kSampleAllBelow = 1024;  // windows shorter than this are looked at whole
constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kBK = 64;
constexpr uint32_t kStageABytes = kBM * kBK * 2;
constexpr uint32_t kStageBBytes = kBN * kBK * 2;
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr int kAcc = 4;       // TMEM accumulators of kBN columns, one per epilogue warpgroup
constexpr int kEpiWarps = 4 * kAcc;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = 64 + kEpiThreads;
static_assert(kBinWords * kBM == kEpiThreads * 32, "pass 3 staging fills the histogram space");

struct __align__(1024) Smem {
  uint8_t a[kStages][kStageABytes];
  uint8_t b[kStages][kStageBBytes];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[kAcc];
  uint64_t acc_empty[kAcc];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  // per row (column) histogram of pass 2; pass 3 reuses the space to stage scores
  // (bins 2w and 2w+1 of a row share word w: low and high 16 bits; a window holds fewer
  // than 65536 scores, so a count never reaches the other half)
  __align__(16) uint32_t hist[kBinWords][kBM];
  float part_mx[kAcc][kBM];   // pass 1 partial maxima of the warpgroups
  int emit_cnt[kAcc][kBM];    // pass 3 entries each warpgroup emitted, per row
};

__device__ __forceinline__ void on_timeout(Smem& s, uint32_t* status) {
  *reinterpret_cast<volatile int*>(&s.abort) = 1;
  raise_flag(status, RECE_DEVICE_TIMEOUT);
}

struct ItemGeom {
  int r;
  int64_t p0;   // first sorted row of the tile
  int64_t U0;   // union window [U0, U1) in sorted catalogue positions
  int nt;       // kBN-wide tiles covering it
};

// One more count in bin b of the row whose column of words starts at shared address hcol.
__device__ __forceinline__ void bin_add(uint32_t hcol, uint32_t b) {
  const uint32_t addr = hcol + (b >> 1) * (kBM * 4);
  const uint32_t inc = 1u << ((b & 1u) << 4);
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(addr), "r"(inc));
}


__device__ __forceinline__ int64_t chunk_of(int64_t p, int64_t M, int n_c) {
  return (p * n_c) / M;
}

__device__ __forceinline__ ItemGeom item_geom(int64_t item, int64_t tiles_per_round, int64_t N,
                                              int64_t C, int n_c, int n_ec) {
  ItemGeom g;
  g.r = int(item / tiles_per_round);
  g.p0 = (item % tiles_per_round) * kBM;
  const int64_t last = (g.p0 + kBM - 1 < N - 1) ? g.p0 + kBM - 1 : N - 1;
  const int64_t cf = chunk_of(g.p0, N, n_c), cl = chunk_of(last, N, n_c);
  g.U0 = chunk_start(cf - n_ec < 0 ? 0 : cf - n_ec, C, n_c);
  const int64_t U1 = chunk_start(cl + n_ec + 1 > n_c ? n_c : cl + n_ec + 1, C, n_c);
  g.nt = int((U1 - g.U0 + kBN - 1) / kBN);
  return g;
}

__global__ void __launch_bounds__(kThreads, 1) k_select_tc(
    const __grid_constant__ CUtensorMap tmXs, const __grid_constant__ CUtensorMap tmYs,
    int64_t N, int64_t C, int d, int n_c, int n_ec, int n_r, int Qw, int E,
    int2* __restrict__ list, int4* __restrict__ list_count, float* __restrict__ list_theta,
    uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tiles_per_round = (N + kBM - 1) / kBM;
  const int64_t items = tiles_per_round * n_r;
  const int nk = d / kBK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < kAcc; ++i) {
      mbar_init(&s.acc_full[i], 1);
      mbar_init(&s.acc_empty[i], 4);  // the 4 warps of the warpgroup that owns it
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
    if (lane == 0) {
      prefetch_tmap(&tmXs);
      prefetch_tmap(&tmYs);
      uint32_t it = 0;
      for (int64_t item = blockIdx.x; item < items && !*abortp; item += gridDim.x) {
        const ItemGeom g = item_geom(item, tiles_per_round, N, C, n_c, n_ec);
        const int32_t arow = int32_t(int64_t(g.r) * N + g.p0);
        for (int pass = 0; pass < kPasses && !*abortp; ++pass) {
          for (int t = 0; t < g.nt && !*abortp; ++t) {
            const int32_t brow = int32_t(int64_t(g.r) * C + g.U0 + int64_t(t) * kBN);
            for (int ks = 0; ks < nk; ++ks, ++it) {
              const int st = it % kStages;
              if (!mbar_wait(&s.empty[st], ((it / kStages) & 1u) ^ 1u, &s.abort, kTimeoutNs)) {
                on_timeout(s, status);
                break;
              }
              mbar_arrive_expect_tx(&s.full[st], kStageABytes + kStageBBytes);
              tma_load_2d(s.a[st], &tmXs, &s.full[st], ks * kBK, arow);
              tma_load_2d(s.b[st], &tmYs, &s.full[st], ks * kBK, brow);
            }
          }
        }
      }
      for (uint32_t j = (it > kStages ? it - kStages : 0); j < it; ++j)
        mbar_wait_limit(&s.full[j % kStages], (j / kStages) & 1u, kTimeoutNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, kBN);
      uint32_t it = 0, acc_it = 0;
      bool ok = true;
      for (int64_t item = blockIdx.x; item < items && ok && !*abortp; item += gridDim.x) {
        const ItemGeom g = item_geom(item, tiles_per_round, N, C, n_c, n_ec);
        for (int tt = 0; tt < kPasses * g.nt && ok; ++tt, ++acc_it) {
          const int a = acc_it % kAcc;
          if (!mbar_wait(&s.acc_empty[a], ((acc_it / kAcc) & 1u) ^ 1u, &s.abort, kTimeoutNs)) {
            on_timeout(s, status);
            ok = false;
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
      mma_commit(&s.drain);
      mbar_wait_limit(&s.drain, 0, kTimeoutNs);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    // Warpgroup wg owns TMEM accumulator wg, i.e. every kAcc-th tile; each row has one
    // thread in each warpgroup, combined through shared memory at pass boundaries, and
    // each warpgroup fills its own sub-list of the row (no shared counter).
    const int wg = (warp - 2) >> 2;
    const int q4 = warp & 3;  // TMEM lane quarter this warp may access
    const int row_local = q4 * 32 + lane;
    const int et = threadIdx.x - 64;  // epilogue thread 0..kEpiThreads-1
    const uint32_t hcol = smem_u32(&s.hist[0][row_local]);
    // pass 3 staging of this thread's 32 scores (the histogram's space, free by then);
    // 16-byte slot j of the thread sits at j ^ (et & 7): conflict-free vector stores
    float* stage = reinterpret_cast<float*>(&s.hist[0][0]) + et * 32;
    const int swz = et & 7;
    uint32_t acc_it = 0;
    bool ok = true;
    for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
      const ItemGeom g = item_geom(item, tiles_per_round, N, C, n_c, n_ec);
      const int64_t p = g.p0 + row_local;
      const bool valid = p < N;
      int32_t w0 = 0, w1 = 0;  // this row's window, in sorted catalogue positions (< C)
      if (valid) {
        const int64_t c = chunk_of(p, N, n_c);
        w0 = int32_t(chunk_start(c - n_ec < 0 ? 0 : c - n_ec, C, n_c));
        w1 = int32_t(chunk_start(c + n_ec + 1 > n_c ? n_c : c + n_ec + 1, C, n_c));
      }
      // pass 1 looks at the first 32 columns of every tile (a strided quarter of the
      // window) unless the window is short, then at all of it
      const bool sample_all = w1 - w0 < kSampleAllBelow;
      const bool histo = valid && w1 - w0 > E;  // else every window score is emitted
      float mx = -INFINITY;  // pass 1: max of the looked-at scores
      BinMap bmap{0u, 0u, 0u};
      float thr = -INFINITY;  // pass 3 emits a score iff score >= thr
      int2* out = list + ((int64_t(g.r) * N + (valid ? p : 0)) * kAcc + wg) * Qw;
      int emitted = 0;
      for (int pass = 0; pass < kPasses; ++pass) {
        if (pass == 1) {
          // combine the warpgroups' maxima; reset this item's histogram
          named_barrier(1, kEpiThreads);
          s.part_mx[wg][row_local] = mx;
          for (int b = wg * (kBinWords / kAcc); b < (wg + 1) * (kBinWords / kAcc); ++b)
            s.hist[b][row_local] = 0;
          named_barrier(1, kEpiThreads);
          mx = s.part_mx[0][row_local];
#pragma unroll
          for (int w = 1; w < kAcc; ++w) mx = fmaxf(mx, s.part_mx[w][row_local]);
          bmap = bin_map(mx, uint32_t(kHeadBins));
        } else if (pass == 2) {
          named_barrier(1, kEpiThreads);  // every histogram increment has landed
          if (histo) {  // else thr stays -inf: emit the whole window
            // the smallest bin b* (< 255, the last one open) whose cumulative count
            // reaches E: whole blocks of 16 bins are skipped while their sum falls short
            uint32_t cum = 0;
            for (int w0 = 0; w0 < kBinWords; w0 += 8) {
              uint32_t blk = 0;
#pragma unroll
              for (int w = 0; w < 8; ++w) {
                const uint32_t v = s.hist[w0 + w][row_local];
                blk += (v & 0xFFFFu) + (v >> 16);
              }
              if (cum + blk < uint32_t(E)) {
                cum += blk;
                continue;
              }
              int bstar = -1;
              for (int b = 2 * w0; b < 2 * w0 + 16 && b < kBins - 1; ++b) {
                cum += (s.hist[b >> 1][row_local] >> ((b & 1) * 16)) & 0xFFFFu;
                if (cum >= uint32_t(E)) {
                  bstar = b;
                  break;
                }
              }
              if (bstar >= 0) thr = cut_threshold(bmap, uint32_t(bstar + 1) << 20);
              break;
            }
          }
          named_barrier(1, kEpiThreads);  // histogram read by all: its space is staging now
        }
        for (int t = 0; t < g.nt; ++t, ++acc_it) {
          const int a = acc_it % kAcc;
          if (a != wg) continue;  // another warpgroup's tile
          if (!ok || !mbar_wait(&s.acc_full[a], (acc_it / kAcc) & 1u, &s.abort, kTimeoutNs)) {
            if (ok) on_timeout(s, status);
            ok = false;
            continue;  // keep the loop structure so every barrier is still met
          }
          tc_fence_after();
          const int32_t q0 = int32_t(g.U0) + t * kBN;  // sorted positions are < C < 2^31
          const uint32_t taddr = tmem + (uint32_t(q4 * 32) << 16) + uint32_t(a * kBN);
#pragma unroll 1
          for (int c0 = 0; c0 < kBN; c0 += 32) {
            const int32_t qa = q0 + c0;
            const bool need = valid && qa < w1 && qa + 32 > w0 &&
                              (pass != 0 || c0 == 0 || sample_all) && (pass != 1 || histo);
            if (!__any_sync(0xFFFFFFFFu, need)) continue;
            float v[32];
            tmem_load32(taddr + c0, v);
            if (!need) continue;
            const int lo = w0 > qa ? w0 - qa : 0, hi = w1 < qa + 32 ? w1 - qa : 32;
            const bool full = lo == 0 && hi == 32;
            if (pass == 0) {
              if (full) {
                float m4[4] = {mx, v[0], v[1], v[2]};
#pragma unroll
                for (int u = 3; u < 32; ++u) m4[u & 3] = fmaxf(m4[u & 3], v[u]);
                mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
              } else {
#pragma unroll
                for (int u = 0; u < 32; ++u)
                  if (u >= lo && u < hi) mx = fmaxf(mx, v[u]);
              }
            } else if (pass == 1) {
              if (full) {
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                  const uint32_t raw = (__float_as_uint(v[u]) * bmap.sig + bmap.off) >> 20;
                  bin_add(hcol, min(raw, uint32_t(kBins - 1)));
                }
              } else {
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                  if (u < lo || u >= hi) continue;
                  const uint32_t raw = (__float_as_uint(v[u]) * bmap.sig + bmap.off) >> 20;
                  bin_add(hcol, min(raw, uint32_t(kBins - 1)));
                }
              }
            } else {
              // the bit mask of passing columns (four independent partial masks), then one
              // step per set bit
              uint32_t mk[4] = {0u, 0u, 0u, 0u};
#pragma unroll
              for (int u = 0; u < 32; ++u) mk[u & 3] |= (v[u] >= thr ? 1u : 0u) << u;
              uint32_t mask = (mk[0] | mk[1]) | (mk[2] | mk[3]);
              if (!full) mask &= (hi == 32 ? 0xFFFFFFFFu : (1u << hi) - 1u) & ~((1u << lo) - 1u);
              if (mask) {
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  *reinterpret_cast<float4*>(stage + 4 * (j ^ swz)) =
                      make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                do {
                  const int u = __ffs(mask) - 1;
                  mask &= mask - 1u;
                  const float val = stage[4 * ((u >> 2) ^ swz) + (u & 3)];
                  if (emitted < Qw) out[emitted] = make_int2(__float_as_int(val), qa + u);
                  ++emitted;
                } while (mask);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s.acc_empty[a]);
        }
      }
      s.emit_cnt[wg][row_local] = emitted;
      named_barrier(1, kEpiThreads);
      if (wg == 0 && ok && valid) {
        list_count[int64_t(g.r) * N + p] = make_int4(s.emit_cnt[0][row_local], s.emit_cnt[1][row_local],
                                                     s.emit_cnt[2][row_local], s.emit_cnt[3][row_local]);
        list_theta[int64_t(g.r) * N + p] = thr == -INFINITY ? -INFINITY : value_below(thr);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// Capacity of each warpgroup's sub-list of a (round, row): a warpgroup sees a quarter of
// the window, so k + 32 leaves wide room above its share of the ~k emitted scores.
int tc_sublist_capacity(int k) { return k + 32; }
int tc_list_capacity(int k) { return kAcc * tc_sublist_capacity(k); }
// k + 1: the positive may be among the emitted, and k others still give the exactness
// check its margin (see the file comment).
int tc_emit_target(int k) { return k + 1; }

cudaError_t launch_select_tc(const rece_plan_s& p, const void* Xs, const void* Ys, int2* list,
                             int4* list_count, float* list_theta, uint32_t* status,
                             cudaStream_t st) {
  const auto& c = p.cfg;
  if (c.N == 0) return cudaSuccess;
  CUtensorMap tmXs, tmYs;
  cudaError_t e = make_tmap_bf16(&tmXs, Xs, uint64_t(c.n_r) * c.N, c.d, kBM);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tmYs, Ys, uint64_t(c.n_r) * c.C, c.d, kBN);
  if (e != cudaSuccess) return e;
  const int64_t items = ceil_div(c.N, kBM) * c.n_r;
  const int grid = int(items < sm_count() ? items : sm_count());
  const size_t smem = sizeof(Smem) + 1024;
  e = cudaFuncSetAttribute(k_select_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  k_select_tc<<<grid, kThreads, smem, st>>>(tmXs, tmYs, c.N, c.C, c.d, c.n_c, c.n_ec, c.n_r,
                                            tc_sublist_capacity(c.k), tc_emit_target(c.k), list,
                                            list_count, list_theta, status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace rece
