// select_tc.cu -- steps 3-4 on the tcgen05 tensor cores (bf16 mode): chunk-window scores
// (RECE, section 3, Algorithm 1: chunk sets, neighbour window, chunk logits; the rounds
// paragraph) and the candidates for each row's top-k negatives (SCE abstract).
//
// Work item = (round r, 128 consecutive sorted rows).  Their chunks' windows are a
// contiguous range of sorted catalogue rows (the union of the windows), streamed by TMA in
// 128-row tiles aligned to multiples of 128 rows of the sorted copy (positions outside a
// row's own window -- before it, after it, or of another round -- are masked out);
// tcgen05.mma forms the 128 x 128 score tile in TMEM and each row's thread reads its row
// of the tile.  Scores never reach HBM.  Two kernels share the code:
//
// Sampled kernel (the one that normally runs): one pass over the whole window.
//   pass 0  per row: max m of the scores of a sample of its window: the first 16
//           positions of every 128-position tile (1/8 of the window, spread over all of
//           it).  A sampled 128-column tile is one TMA load of 8 boxes of 16 rows (a
//           3-D view of the sorted copy), multiplied like any other tile;
//   pass 1  per row: exact histogram of the sample's scores by distance below an anchor
//           two binades above m (8 bins per binade over 32 binades, tc_bins.cuh);
//           the lower edge t0 of the bin where the count from the top reaches
//           m_s = E' + 4.5 sqrt(E') + 1 (E' = E times the sample's share of the window,
//           E = k + 1) is a threshold that, but with probability ~1e-5, at least E of
//           the window's scores pass;
//   pass 2  the whole window: every score >= t0 is emitted as (score, sorted position)
//           into the row's list and counted in a 32-bin histogram of its distance above
//           t0 (1/8 binade per bin, the last bin open).  From that histogram the row's
//           exact cut t* >= t0 -- the highest bin edge with at least E emitted scores at
//           or above it -- is recorded as theta = the largest fp32 value below t*: the
//           merge keeps only the entries above theta, and no score it did not see can
//           be above theta.
//   A row for which fewer than E scores passed t0 (the sample misled) or whose list
//   overflowed cannot be certified; its item is appended to a redo list.
// Exact kernel (the redo list's items; it rewrites their lists): three passes with the
//   threshold found without any assumption on the scores' distribution:
//   pass 0  per row: max m of a strided quarter of its window's scores (the first 32
//           columns of every tile; all of them when the window is short);
//   pass 1  exact histogram of all the window's scores below an anchor two binades
//           above m;
//   pass 2  the smallest bin b* whose cumulative count reaches E sets the cut t at
//           its lower edge; every score >= t is emitted (equal scores share a bin, so a
//           tie is never split); theta = the largest fp32 value below t.
// Each of the four epilogue warpgroups (one per 128-column TMEM accumulator, every fourth
// tile) writes its own sub-list of the row, up to k + 32 entries, and its count of all that
// passed; both kernels give every warpgroup the same tiles, so a row's kept entries come
// out in the same order whichever kernel wrote its list.  The merge kernel keeps the k
// best; the selection is exact whenever no list overflowed and every round's theta is
// below the k-th kept score, which the merge checks row by row.  Without an overflow the
// check always passes: the round with the highest cut has at least E = k + 1 entries at
// or above it, at least k of them negatives and none of them a duplicate that an earlier
// round left out (that round's cut would be higher still), so the k-th kept score is >=
// every round's cut.
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
constexpr int kHeadBins = 16;          // bins above the pass 0 max (2 binades)
constexpr int kSampleAllBelow = 1024;  // exact kernel: windows shorter are looked at whole
constexpr int kFineBins = 32;          // sampled kernel: bins of the emitted scores above t0
constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kBK = 64;
constexpr int kSampleRun = 16;                  // sampled positions per 128-position tile
constexpr int kSampleGroups = kBN / kSampleRun; // tiles one sampled 128-column tile covers
constexpr uint32_t kStageABytes = kBM * kBK * 2;
constexpr uint32_t kStageBBytes = kBN * kBK * 2;
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr int kAcc = 4;       // TMEM accumulators of kBN columns, one per epilogue warpgroup
constexpr int kEpiWarps = 4 * kAcc;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = 64 + kEpiThreads;
static_assert(kBinWords * kBM == kEpiThreads * 32, "emission staging fills the histogram space");

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
  int redo;  // sampled kernel: a row of the current item could not be certified
  // per row (column) histogram of pass 1; pass 2 reuses the space to stage scores
  // (bins 2w and 2w+1 of a row share word w: low and high 16 bits; a window holds fewer
  // than 65536 scores, so a count never reaches the other half)
  __align__(16) uint32_t hist[kBinWords][kBM];
  uint32_t fine[kFineBins / 2][kBM];  // sampled kernel, pass 2: bins above t0, 16-bit counts
  float part_mx[kAcc][kBM];   // pass 0 partial maxima of the warpgroups
  int emit_cnt[kAcc][kBM];    // pass 2 entries each warpgroup emitted, per row
};

__device__ __forceinline__ void on_timeout(Smem& s, uint32_t* status) {
  *reinterpret_cast<volatile int*>(&s.abort) = 1;
  raise_flag(status, RECE_DEVICE_TIMEOUT);
}

struct ItemGeom {
  int r;
  int64_t p0;   // first sorted row of the tile
  int64_t g0;   // first 128-row group of the sorted copy (all rounds' rows in a row)
                // that the union window of the tile's rows touches
  int nt;       // 128-row groups covering the union window
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
  const int64_t U0 = chunk_start(cf - n_ec < 0 ? 0 : cf - n_ec, C, n_c);
  const int64_t U1 = chunk_start(cl + n_ec + 1 > n_c ? n_c : cl + n_ec + 1, C, n_c);
  const int64_t f0 = int64_t(g.r) * C + U0, f1 = int64_t(g.r) * C + U1;
  g.g0 = f0 / kBN;
  g.nt = int((f1 + kBN - 1) / kBN - g.g0);
  return g;
}

// Bits i < 16 of the run of positions q, q+1, ..., q+15 that lie in [w0, w1).
__device__ __forceinline__ uint32_t run_mask16(int32_t q, int32_t w0, int32_t w1) {
  int32_t lo = w0 - q, hi = w1 - q;
  lo = lo < 0 ? 0 : (lo > 16 ? 16 : lo);
  hi = hi < 0 ? 0 : (hi > 16 ? 16 : hi);
  return hi > lo ? ((1u << hi) - 1u) & ~((1u << lo) - 1u) : 0u;
}

// Sampled positions (the first kSampleRun of every 128-row group of the sorted copy)
// among the first f rows of the copy.
__device__ __forceinline__ int64_t sampled_below(int64_t f) {
  const int64_t rem = f % kBN;
  return (f / kBN) * kSampleRun + (rem < kSampleRun ? rem : kSampleRun);
}

// Order-preserving integer image of an fp32 value, and back.
__device__ __forceinline__ uint32_t ord_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float ord_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// The smallest bin b* (< kBins - 1, the last one open) of the row's histogram column
// whose cumulative count reaches `want`, or -1.  Whole blocks of 16 bins are skipped
// while their sum falls short.
__device__ __forceinline__ int cut_bin(const uint32_t (&hist)[kBinWords][kBM], int row,
                                       uint32_t want) {
  uint32_t cum = 0;
  for (int w0 = 0; w0 < kBinWords; w0 += 8) {
    uint32_t blk = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const uint32_t v = hist[w0 + w][row];
      blk += (v & 0xFFFFu) + (v >> 16);
    }
    if (cum + blk < want) {
      cum += blk;
      continue;
    }
    for (int b = 2 * w0; b < 2 * w0 + 16 && b < kBins - 1; ++b) {
      cum += (hist[b >> 1][row] >> ((b & 1) * 16)) & 0xFFFFu;
      if (cum >= want) return b;
    }
    return -1;
  }
  return -1;
}

// Work items come from the range [0, n_r * ceil(N / 128)) or, for the exact kernel run
// on the sampled kernel's failures, from items_list[0 .. *items_count).
template <bool kSampled>
__global__ void __launch_bounds__(kThreads, 1) k_select_tc(
    const __grid_constant__ CUtensorMap tmXs, const __grid_constant__ CUtensorMap tmYs,
    const __grid_constant__ CUtensorMap tmYsS, int64_t N, int64_t C, int d, int n_c, int n_ec,
    int n_r, int Qw, int E, int2* __restrict__ list, int4* __restrict__ list_count,
    float* __restrict__ list_theta, const int32_t* __restrict__ items_list,
    const uint32_t* items_count, int32_t* __restrict__ redo_list, uint32_t* redo_count,
    uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                     ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tiles_per_round = (N + kBM - 1) / kBM;
  const int64_t items = items_list ? int64_t(*reinterpret_cast<const volatile uint32_t*>(items_count))
                                   : tiles_per_round * n_r;
  const int nk = d / kBK;
  auto item_at = [&](int64_t i) -> int64_t { return items_list ? int64_t(items_list[i]) : i; };
  // tiles of pass `pass` of an item whose union window spans nt groups: the sampled
  // kernel's passes 0 and 1 read 8 groups per tile
  auto pass_tiles = [&](int pass, int nt) {
    return (kSampled && pass < 2) ? (nt + kSampleGroups - 1) / kSampleGroups : nt;
  };
  if (items == 0) return;  // (the redo launch when nothing failed: no barrier, no TMEM)

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
    s.redo = 0;
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
      if (kSampled) prefetch_tmap(&tmYsS);
      uint32_t it = 0;
      for (int64_t i = blockIdx.x; i < items && !*abortp; i += gridDim.x) {
        const ItemGeom g = item_geom(item_at(i), tiles_per_round, N, C, n_c, n_ec);
        const int32_t arow = int32_t(int64_t(g.r) * N + g.p0);
        for (int pass = 0; pass < kPasses && !*abortp; ++pass) {
          const bool spass = kSampled && pass < 2;
          const int ntp = pass_tiles(pass, g.nt);
          for (int t = 0; t < ntp && !*abortp; ++t) {
            for (int ks = 0; ks < nk; ++ks, ++it) {
              const int st = it % kStages;
              if (!mbar_wait(&s.empty[st], ((it / kStages) & 1u) ^ 1u, &s.abort, kTimeoutNs)) {
                on_timeout(s, status);
                break;
              }
              mbar_arrive_expect_tx(&s.full[st], kStageABytes + kStageBBytes);
              tma_load_2d(s.a[st], &tmXs, &s.full[st], ks * kBK, arow);
              if (spass)  // rows 0..15 of groups g0 + 8t .. g0 + 8t + 7
                tma_load_3d(s.b[st], &tmYsS, &s.full[st], ks * kBK, 0,
                            int32_t(g.g0 + int64_t(t) * kSampleGroups));
              else
                tma_load_2d(s.b[st], &tmYs, &s.full[st], ks * kBK,
                            int32_t((g.g0 + t) * kBN));
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
      for (int64_t i = blockIdx.x; i < items && ok && !*abortp; i += gridDim.x) {
        const ItemGeom g = item_geom(item_at(i), tiles_per_round, N, C, n_c, n_ec);
        int tiles = 0;
        for (int pass = 0; pass < kPasses; ++pass) tiles += pass_tiles(pass, g.nt);
        for (int tt = 0; tt < tiles && ok; ++tt, ++acc_it) {
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
    const uint32_t fcol = smem_u32(&s.fine[0][row_local]);
    // emission staging of this thread's 32 scores (the histogram's space, free by then);
    // 16-byte slot j of the thread sits at j ^ (et & 7): conflict-free vector stores
    float* stage = reinterpret_cast<float*>(&s.hist[0][0]) + et * 32;
    const int swz = et & 7;
    uint32_t acc_it = 0;
    bool ok = true;
    for (int64_t i = blockIdx.x; i < items; i += gridDim.x) {
      const int64_t item = item_at(i);
      const ItemGeom g = item_geom(item, tiles_per_round, N, C, n_c, n_ec);
      const int64_t p = g.p0 + row_local;
      const bool valid = p < N;
      const int64_t rC = int64_t(g.r) * C;
      int32_t w0 = 0, w1 = 0;  // this row's window, in sorted catalogue positions (< C)
      if (valid) {
        const int64_t c = chunk_of(p, N, n_c);
        w0 = int32_t(chunk_start(c - n_ec < 0 ? 0 : c - n_ec, C, n_c));
        w1 = int32_t(chunk_start(c + n_ec + 1 > n_c ? n_c : c + n_ec + 1, C, n_c));
      }
      // exact kernel, pass 0: the first 32 columns of every tile (a strided quarter of
      // the window) unless the window is short, then all of it
      const bool sample_all = kSampled || w1 - w0 < kSampleAllBelow;
      // how many scores the cut of pass 1's histogram must leave above it, and whether
      // a cut is sought at all (else every window score is emitted)
      uint32_t want = uint32_t(E);
      bool histo = valid && w1 - w0 > E;
      if (kSampled && histo) {
        const float ws = float(sampled_below(rC + w1) - sampled_below(rC + w0));
        const float e1 = float(E) * ws / float(w1 - w0);
        const float m = ceilf(e1 + 4.5f * sqrtf(e1)) + 1.0f;
        histo = m < ws;
        want = uint32_t(m);
      }
      float mx = -INFINITY;  // pass 0: max of the looked-at scores
      BinMap bmap{0u, 0u, 0u};
      float thr = -INFINITY;  // pass 2 emits a score iff score >= thr
      uint32_t thr_key = ord_key(-INFINITY);
      int2* out = list + ((int64_t(g.r) * N + (valid ? p : 0)) * kAcc + wg) * Qw;
      int emitted = 0;
      for (int pass = 0; pass < kPasses; ++pass) {
        const bool spass = kSampled && pass < 2;
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
            const int bstar = cut_bin(s.hist, row_local, want);
            if (bstar >= 0) thr = cut_threshold(bmap, uint32_t(bstar + 1) << 20);
          }
          // a zero threshold as -0: every score that passes it (+0 and -0 included) then
          // has an order key at or above thr_key, so the fine bins below never wrap
          if (thr == 0.0f) thr = -0.0f;
          thr_key = ord_key(thr);
          if (kSampled && wg == 0)
            for (int b = 0; b < kFineBins / 2; ++b) s.fine[b][row_local] = 0;
          named_barrier(1, kEpiThreads);  // histogram read by all: its space is staging now
        }
        const int ntp = pass_tiles(pass, g.nt);
        for (int t = 0; t < ntp; ++t, ++acc_it) {
          const int a = acc_it % kAcc;
          if (a != wg) continue;  // another warpgroup's tile
          if (!ok || !mbar_wait(&s.acc_full[a], (acc_it / kAcc) & 1u, &s.abort, kTimeoutNs)) {
            if (ok) on_timeout(s, status);
            ok = false;
            continue;  // keep the loop structure so every barrier is still met
          }
          tc_fence_after();
          const uint32_t taddr = tmem + (uint32_t(q4 * 32) << 16) + uint32_t(a * kBN);
#pragma unroll 1
          for (int c0 = 0; c0 < kBN; c0 += 32) {
            // sorted positions of the chunk's columns: two runs of 16 (groups 2c0/32 and
            // 2c0/32 + 1 of a sampled tile; consecutive in a full one); positions are
            // round-local and may fall outside [0, C) at a round's ends
            int32_t qa, qb;
            if (spass) {
              qa = int32_t((g.g0 + int64_t(t) * kSampleGroups + (c0 >> 4)) * kBN - rC);
              qb = qa + kBN;
            } else {
              qa = int32_t((g.g0 + t) * kBN + c0 - rC);
              qb = qa + 16;
            }
            const uint32_t win =
                valid ? run_mask16(qa, w0, w1) | (run_mask16(qb, w0, w1) << 16) : 0u;
            const bool need = win != 0u && (pass != 0 || c0 == 0 || sample_all) &&
                              (pass != 1 || histo);
            if (!__any_sync(0xFFFFFFFFu, need)) continue;
            float v[32];
            tmem_load32(taddr + c0, v);
            if (!need) continue;
            const bool full = win == 0xFFFFFFFFu;
            if (pass == 0) {
              if (full) {
                float m4[4] = {mx, v[0], v[1], v[2]};
#pragma unroll
                for (int u = 3; u < 32; ++u) m4[u & 3] = fmaxf(m4[u & 3], v[u]);
                mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
              } else {
#pragma unroll
                for (int u = 0; u < 32; ++u)
                  if ((win >> u) & 1u) mx = fmaxf(mx, v[u]);
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
                  if (!((win >> u) & 1u)) continue;
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
              uint32_t mask = ((mk[0] | mk[1]) | (mk[2] | mk[3])) & win;
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
                  if (kSampled) {
                    const uint32_t fb = (ord_key(val) - thr_key) >> 20;
                    bin_add(fcol, fb < kFineBins - 1 ? fb : uint32_t(kFineBins - 1));
                  }
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
        const int4 cnt = make_int4(s.emit_cnt[0][row_local], s.emit_cnt[1][row_local],
                                   s.emit_cnt[2][row_local], s.emit_cnt[3][row_local]);
        float theta = thr == -INFINITY ? -INFINITY : value_below(thr);
        if (kSampled) {
          // the exact cut among the emitted scores: the highest bin edge of the fine
          // histogram with at least E of them at or above it
          const bool over = cnt.x > Qw || cnt.y > Qw || cnt.z > Qw || cnt.w > Qw;
          bool fail = over;
          if (thr != -INFINITY) {
            uint32_t total = 0;
#pragma unroll
            for (int b = 0; b < kFineBins / 2; ++b) {
              const uint32_t w = s.fine[b][row_local];
              total += (w & 0xFFFFu) + (w >> 16);
            }
            if (total < uint32_t(E)) {
              fail = true;  // the sample put t0 above the E-th score
            } else {
              // the largest b with at least E emitted scores in bins b and above
              uint32_t below = 0;
              int b = 0;
              for (; b + 1 < kFineBins; ++b) {
                const uint32_t cb = (s.fine[b >> 1][row_local] >> ((b & 1) * 16)) & 0xFFFFu;
                if (total - (below + cb) < uint32_t(E)) break;
                below += cb;
              }
              theta = value_below(b == 0 ? thr : ord_float(thr_key + (uint32_t(b) << 20)));
            }
          }
          if (fail) s.redo = 1;
        }
        list_count[int64_t(g.r) * N + p] = cnt;
        list_theta[int64_t(g.r) * N + p] = theta;
      }
      if (kSampled) {
        named_barrier(1, kEpiThreads);
        if (et == 0 && s.redo) {
          s.redo = 0;
          redo_list[atomicAdd(redo_count, 1u)] = int32_t(item);
        }
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
// the window's tiles, so k + 32 leaves wide room above its share of what passes t0
// (about 1.3 to 1.8 times k in all; a row that overflows goes to the exact kernel).
int tc_sublist_capacity(int k) { return k + 32; }
int tc_list_capacity(int k) { return kAcc * tc_sublist_capacity(k); }
// k + 1: the positive may be among the emitted, and k others still give the exactness
// check its margin (see the file comment).
int tc_emit_target(int k) { return k + 1; }
// Rows of the sorted copy Ys a tensor map may reach: whole 128-row groups.
int64_t tc_ys_rows(int64_t rows) { return ceil_div(rows, kBN) * kBN; }
int64_t tc_select_items(const rece_plan_s& p) { return ceil_div(p.cfg.N, kBM) * p.cfg.n_r; }

cudaError_t launch_select_tc(const rece_plan_s& p, const void* Xs, const void* Ys, int2* list,
                             int4* list_count, float* list_theta, int32_t* redo_list,
                             uint32_t* redo_count, uint32_t* status, cudaStream_t st) {
  const auto& c = p.cfg;
  if (c.N == 0) return cudaSuccess;
  CUtensorMap tmXs, tmYs, tmYsS;
  cudaError_t e = make_tmap_bf16(&tmXs, Xs, uint64_t(c.n_r) * c.N, c.d, kBM);
  if (e != cudaSuccess) return e;
  // the sorted copy of all rounds as whole 128-row groups (the copy is padded to them):
  // full tiles of 128 rows, and sampled tiles of the first 16 rows of 8 groups each
  const uint64_t groups = uint64_t(tc_ys_rows(int64_t(c.n_r) * c.C) / kBN);
  e = make_tmap_bf16(&tmYs, Ys, groups * kBN, c.d, kBN);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16_groups(&tmYsS, Ys, c.d, groups, kBN, kSampleRun, kSampleGroups);
  if (e != cudaSuccess) return e;
  const int64_t items = tc_select_items(p);
  const int grid = int(items < sm_count() ? items : sm_count());
  const size_t smem = sizeof(Smem) + 1024;
  e = cudaFuncSetAttribute(k_select_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(smem));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_select_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(smem));
  if (e != cudaSuccess) return e;
  if (!p.tc_sampled) {  // the exact kernel over every item
    k_select_tc<false><<<grid, kThreads, smem, st>>>(
        tmXs, tmYs, tmYsS, c.N, c.C, c.d, c.n_c, c.n_ec, c.n_r, tc_sublist_capacity(c.k),
        tc_emit_target(c.k), list, list_count, list_theta, nullptr, nullptr, nullptr, nullptr,
        status);
    count_launches(1);
    return cudaGetLastError();
  }
  e = cudaMemsetAsync(redo_count, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  k_select_tc<true><<<grid, kThreads, smem, st>>>(
      tmXs, tmYs, tmYsS, c.N, c.C, c.d, c.n_c, c.n_ec, c.n_r, tc_sublist_capacity(c.k),
      tc_emit_target(c.k), list, list_count, list_theta, nullptr, nullptr, redo_list,
      redo_count, status);
  count_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the items the sampled kernel could not certify, again with the exact kernel (a grid
  // that returns at once when the list is empty)
  k_select_tc<false><<<grid, kThreads, smem, st>>>(
      tmXs, tmYs, tmYsS, c.N, c.C, c.d, c.n_c, c.n_ec, c.n_r, tc_sublist_capacity(c.k),
      tc_emit_target(c.k), list, list_count, list_theta, redo_list, redo_count, nullptr,
      nullptr, status);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace rece
