// merge_tc.cu -- steps 4-5 for the tensor-core selection: a warp per row (k < 512) or a
// CTA of four warps per row (k >= 512, further down).
//
// The row's candidates are the (score, sorted position) pairs its rounds emitted.  A pair
// of round r is translated to its item j and dropped when j is the row's positive or when
// j also lies in the row's window of an earlier round r' < r (that round saw the same
// pair, so the union of the rounds stays de-duplicated -- the RECE paper's ln(count)
// correction for repeated pairs amounts to counting each pair once).  The k best of the
// rest by (score descending, item ascending) are found with a radix select (digits of
// the score key from its highest varying bit, then the item ids if the k-th place is
// tied), kept in a fixed order (by round, then list order, or sorted position where the
// backward's band products follow), and give the row's loss (RECE, Algorithm 1's loss
// lines):
//   lse_i = log(exp(l+) + sum_j exp(l_j)),  loss_i = lse_i - l+.
// Exactness check: each round recorded the largest score it did not emit; if no list
// overflowed and every such score is below the k-th kept score, nothing left out could
// have been selected.  Rows failing the check are counted in the status area (second
// word) and flagged RECE_DEVICE_INEXACT.
#include "common.cuh"
#include "plan.h"
#include "tc.h"

namespace rece {
namespace {

constexpr int kThreads = 256;
constexpr int kCountBytes = 16 * 32 * 4;  // per-warp digit-count table

// A warp's table: the digit counts, and in grouped mode the bit map of a window (two words
// a slice) and its slice starts, whichever is larger.
__host__ __device__ __forceinline__ size_t merge_table_bytes(bool grouped, int Sp) {
  const size_t g = grouped ? size_t(3) * size_t(Sp) * 4 : 0;
  return g > size_t(kCountBytes) ? (g + 15) / 16 * 16 : size_t(kCountBytes);
}

struct WarpSel {
  uint32_t T;  // threshold key
  int need;    // how many keys equal to T are kept
  int eq;      // how many keys equal T
};

__device__ __forceinline__ uint32_t warp_or(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v |= __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
__device__ __forceinline__ uint32_t warp_and(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v &= __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// The want-th largest (1-based) of the warp's keys in play (get(q, key) -> in play, its
// key; q < n), found four bits at a time from the highest bit in which the keys differ.
// Each lane counts its own keys in its own column of the 16 x 32 table cnt, so no two
// lanes ever update one counter.  On return, the kept set is: every key > T, and `need`
// of the `eq` keys equal to T (all of them when need == eq).  The scan stops early when
// the digit holding the want-th key is wanted whole; T then carries that digit's prefix
// with zero bits below it, and every key of the digit is >= T.
template <typename Get>
__device__ WarpSel warp_select_kth(int n, int want, Get get, uint32_t* cnt) {
  const int lane = threadIdx.x & 31;
  uint32_t orv = 0u, andv = 0xFFFFFFFFu;
  int m = 0;
  for (int q = lane; q < n; q += 32) {
    uint32_t key;
    if (get(q, key)) {
      orv |= key;
      andv &= key;
      ++m;
    }
  }
  orv = warp_or(orv);
  andv = warp_and(andv);
  m = int(warp_sum(float(m)));  // exact: m <= n < 2^24
  const uint32_t diff = orv ^ andv;
  if (diff == 0u) return WarpSel{andv, want, m};
  int shift = ((31 - __clz(diff)) >> 2) << 2;
  uint32_t pmask = shift == 28 ? 0u : ~((1u << (shift + 4)) - 1u);
  uint32_t prefix = andv & pmask;
  const int hb = lane >> 1, hh = lane & 1;
  for (;;) {
#pragma unroll
    for (int b = 0; b < 16; ++b) cnt[b * 32 + lane] = 0u;
    for (int q = lane; q < n; q += 32) {
      uint32_t key;
      if (get(q, key) && (key & pmask) == prefix)
        atomicAdd(&cnt[((key >> shift) & 15u) * 32 + lane], 1u);
    }
    __syncwarp();
    // lanes 2b and 2b+1 add up digit b's 32 columns, half each (rotated: no bank conflict)
    uint32_t s = 0u;
#pragma unroll
    for (int t = 0; t < 16; ++t) s += cnt[hb * 32 + hh * 16 + ((t + hb) & 15)];
    s += __shfl_xor_sync(0xFFFFFFFFu, s, 1);
    // lane l < 16 takes digit 15 - l: digits in descending order along the lanes
    const uint32_t c0 = __shfl_sync(0xFFFFFFFFu, s, (2 * (15 - lane)) & 31);
    const int c = lane < 16 ? int(c0) : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    const int excl = incl - c;
    const bool mine = lane < 16 && excl < want && want <= incl;
    const int src = __ffs(__ballot_sync(0xFFFFFFFFu, mine)) - 1;
    const int above = __shfl_sync(0xFFFFFFFFu, excl, src);
    const int count = __shfl_sync(0xFFFFFFFFu, c, src);
    want -= above;
    prefix |= uint32_t(15 - src) << shift;
    pmask |= 15u << shift;
    __syncwarp();  // the table is cleared again by the next pass
    if (count == want || shift == 0) return WarpSel{prefix, want, count};
    shift -= 4;
  }
}

template <typename T>
struct MergeArgs {
  const T* X;
  const T* Y;
  const int32_t* targets;
  const int32_t* py;
  const int32_t* invX;
  const int32_t* invY;  // sorted position of each item, per round
  const int32_t* chunkY;
  const int2* list;
  const int4* list_count;
  const float* list_theta;
  int64_t N, C;
  int d, k, n_r, n_c, n_ec, Qw, Sp;
  int32_t* selected;
  int2* kept;
  int32_t* kept_off;
  float* pos_logit;
  float* lse_out;
  float* row_loss;
  float* logits;
  uint32_t* status;
  int32_t* spill_rows;    // rows whose candidates did not fit the fast path's buffer
  uint32_t* spill_count;  // how many (status area)
};

// One row, one warp.  keys / poss: the candidate buffer (cap entries each); cnt: the
// warp's 16 x 32 count table (shared memory).  When more candidates arrive than the buffer
// holds, a row with `spill` set is handed to the spill list and nothing is written for it
// (returns false); without, the first cap are kept and the row is flagged inexact.
// kGrouped: also hand the backward's tensor-core dX its data (entries grouped by slice,
// probabilities, the positive logit); else the kept entries go out in list order.
// kGather: candidates per lane gathered together (list entry, then item, then chunk):
// 8 pays at k >= 384, where a round's candidates fill the wider batches; else 4.
template <typename T, bool kGrouped, int kGather>
__device__ __forceinline__ bool merge_row(const MergeArgs<T>& A, int64_t i, uint32_t* cnt,
                                          uint32_t* keys, int32_t* poss, int cap, bool spill) {
  const T* __restrict__ X = A.X;
  const T* __restrict__ Y = A.Y;
  const int32_t* __restrict__ targets = A.targets;
  const int32_t* __restrict__ py = A.py;
  const int32_t* __restrict__ invX = A.invX;
  const int32_t* __restrict__ chunkY = A.chunkY;
  const int2* __restrict__ list = A.list;
  const int4* __restrict__ list_count = A.list_count;
  const float* __restrict__ list_theta = A.list_theta;
  const int64_t N = A.N, C = A.C;
  const int d = A.d, k = A.k, n_r = A.n_r, n_c = A.n_c, n_ec = A.n_ec, Qw = A.Qw, Sp = A.Sp;
  int32_t* __restrict__ selected = A.selected;
  int2* __restrict__ kept = A.kept;
  int32_t* __restrict__ kept_off = A.kept_off;
  float* __restrict__ pos_logit = A.pos_logit;
  float* __restrict__ lse_out = A.lse_out;
  float* __restrict__ row_loss = A.row_loss;
  float* __restrict__ logits = A.logits;
  uint32_t* status = A.status;
  const int lane = threadIdx.x & 31;
  (void)Y;
  const int32_t z = targets[i];
  const bool z_ok = z >= 0 && z < C;

  // gather the candidates of all rounds
  int cx[8], px_of[8];  // per round: the row's chunk and sorted position
  for (int r = 0; r < n_r; ++r) {
    px_of[r] = invX[int64_t(r) * N + i];
    cx[r] = int((int64_t(px_of[r]) * n_c) / N);
  }
  int n = 0;
  int rb[9];           // candidates of round r: [rb[r], rb[r + 1])
  uint32_t kmax = 0u;  // largest key buffered by this lane (0: none)
  bool overflow = false;
  float theta_max = -INFINITY;
  for (int r = 0; r < n_r; ++r) {
    rb[r] = n < cap ? n : cap;
    const int64_t p = invX[int64_t(r) * N + i];
    // four sub-lists (one per epilogue warpgroup of the selection kernel), read as one
    // concatenated list, kGather independent entries per lane in flight at a time
    const int4 c4 = list_count[int64_t(r) * N + p];
    // every entry at or below the round's theta lies below its cut: not a candidate
    const float theta_r = list_theta[int64_t(r) * N + p];
    theta_max = fmaxf(theta_max, theta_r);
    const int cs[4] = {c4.x < Qw ? c4.x : Qw, c4.y < Qw ? c4.y : Qw, c4.z < Qw ? c4.z : Qw,
                       c4.w < Qw ? c4.w : Qw};
    overflow |= c4.x > Qw || c4.y > Qw || c4.z > Qw || c4.w > Qw;
    const int total = cs[0] + cs[1] + cs[2] + cs[3];
    const int2* L = list + (int64_t(r) * N + p) * 4 * Qw;
    for (int a0 = 0; a0 < total; a0 += 32 * kGather) {
      int2 e[kGather];
      int32_t jj[kGather];
      bool in[kGather];
#pragma unroll
      for (int u = 0; u < kGather; ++u) {
        int a = a0 + 32 * u + lane;
        in[u] = a < total;
        int w = 0;
        while (w < 3 && a >= cs[w]) {
          a -= cs[w];
          ++w;
        }
        e[u] = in[u] ? L[w * Qw + a] : make_int2(0, 0);
        in[u] = in[u] && __int_as_float(e[u].x) > theta_r;
      }
#pragma unroll
      for (int u = 0; u < kGather; ++u) jj[u] = in[u] ? py[int64_t(r) * C + e[u].y] : -1;
      bool keep[kGather];
#pragma unroll
      for (int u = 0; u < kGather; ++u) {
        keep[u] = in[u] && jj[u] != z;
        for (int rp = 0; rp < r && keep[u]; ++rp) {
          const int dc = chunkY[int64_t(rp) * C + jj[u]] - cx[rp];
          if (dc >= -n_ec && dc <= n_ec) keep[u] = false;
        }
      }
#pragma unroll
      for (int u = 0; u < kGather; ++u) {
        const unsigned b = __ballot_sync(0xFFFFFFFFu, keep[u]);
        if (keep[u]) {
          const int pos = n + __popc(b & ((1u << lane) - 1u));
          if (pos < cap) {
            const uint32_t key = score_key(__int_as_float(e[u].x));
            keys[pos] = key;
            // grouped output needs the sorted position; otherwise keep the item id, which
            // the output then reads without a second gather
            poss[pos] = kGrouped ? e[u].y : jj[u];
            kmax = key > kmax ? key : kmax;
          }
        }
        n += __popc(b);
      }
    }
  }
  if (n > cap) {  // more candidates than the buffer holds
    if (spill) {
      if (lane == 0) A.spill_rows[atomicAdd(A.spill_count, 1u)] = int32_t(i);
      return false;
    }
    overflow = true;  // keep the first cap, flag the row
    n = cap;
  }
  rb[n_r] = n;
  __syncwarp();

  // the positive's logit
  float part = 0.0f;
  if (z_ok) {
    const T* x = X + i * d;
    const T* y = Y + int64_t(z) * d;
    for (int t = lane; t < d; t += 32) part = fmaf(to_f32(x[t]), to_f32(y[t]), part);
  }
  const float lp = warp_sum(part);

  // item id of candidate q (its round found from the boundaries)
  auto item_of = [&](int q) {
    if constexpr (!kGrouped) return poss[q];
    int r = 0;
    while (r + 1 < n_r && q >= rb[r + 1]) ++r;
    return py[int64_t(r) * C + poss[q]];
  };

  // the k best
  const int kk = k < n ? k : n;
  const bool all = kk >= n;
  WarpSel s1{0u, 0, 0}, s2{0u, 0, 0};
  bool tie = false;
  if (!all) {
    s1 = warp_select_kth(
        n, kk, [&](int q, uint32_t& key) { key = keys[q]; return true; }, cnt);
    if (s1.need != s1.eq) {
      tie = true;
      const uint32_t Tk = s1.T;
      s2 = warp_select_kth(
          n, s1.need,
          [&](int q, uint32_t& key) {
            if (keys[q] != Tk) return false;
            key = ~uint32_t(item_of(q));
            return true;
          },
          cnt);
    }
  }
  // the best candidate is always kept: it bounds the exponentials
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint32_t v = __shfl_xor_sync(0xFFFFFFFFu, kmax, o);
    kmax = v > kmax ? v : kmax;
  }
  const float best = n > 0 ? key_score(kmax) : -INFINITY;
  const float m = fmaxf(lp, best);

  auto take = [&](int a) {
    const uint32_t key = keys[a];
    return all || key > s1.T || (key == s1.T && (!tie || ~uint32_t(item_of(a)) >= s2.T));
  };
  // the row's loss (RECE, Algorithm 1's loss lines); in grouped mode first, so that the
  // kept entries can go out with their softmax probabilities
  float acc = 0.0f, lse = 0.0f;
  if constexpr (kGrouped) {
    for (int a = lane; a < n; a += 32)
      if (take(a)) acc += expf(key_score(keys[a]) - m);
    lse = m + logf(warp_sum(acc) + expf(lp - m));
  }
  // The kept entries, by round and, within a round, in order of sorted position (so
  // grouped by 64-position slice of the round's sorted catalogue): a bit map of the
  // round's window from the start of its first slice, an entry's place being the count of
  // kept positions before it.  Besides the row's outputs (items, logits), the backward
  // gets, indexed by (round, sorted row p): the round's entries
  // kept[r][p][e] = (sorted position, p_ij as two bf16 halves hi | lo << 16, with
  // p_ij = exp(l_ij - lse_i) = bf16(hi) + bf16(lo) to about 16 bits; 0 for a bad target)
  // and the slice starts kept_off[r][p][s] (s = 0..S, entry S = the round's count).
  // The table cnt holds the bit map (2 S words) and the slice starts (S words).
  float* lg = logits ? logits + i * (int64_t(k) + 1) : nullptr;
  int32_t* srow = selected + i * k;
  int ns = 0;
  float worst = INFINITY;
  for (int r = 0; r < n_r; ++r) {
    if constexpr (!kGrouped) {
      // list order: rounds, then each selection warpgroup's emission order
      for (int a0 = rb[r]; a0 < rb[r + 1]; a0 += 32) {
        const int a = a0 + lane;
        const bool tk = a < rb[r + 1] && take(a);
        const unsigned b = __ballot_sync(0xFFFFFFFFu, tk);
        if (tk) {
          const int dest = ns + __popc(b & ((1u << lane) - 1u));
          const float sc = key_score(keys[a]);
          srow[dest] = poss[a];  // the item id (not grouped)
          if (lg) lg[1 + dest] = sc;
          worst = fminf(worst, sc);
          acc += expf(sc - m);
        }
        ns += __popc(b);
      }
      continue;
    }
    const int64_t c = cx[r];
    const int64_t w0 = chunk_start(c - n_ec < 0 ? 0 : c - n_ec, C, n_c);
    const int64_t w1 = chunk_start(c + n_ec + 1 > n_c ? n_c : c + n_ec + 1, C, n_c);
    const int sig0 = int(w0 >> 6);
    const int S = w1 > w0 ? int((w1 - 1) >> 6) - sig0 + 1 : 0;
    const int32_t pbase = sig0 << 6;
    uint32_t* bits = cnt;
    int32_t* soff = reinterpret_cast<int32_t*>(cnt) + 2 * S;
    for (int b = lane; b < 2 * S; b += 32) bits[b] = 0u;
    __syncwarp();
    for (int a = rb[r] + lane; a < rb[r + 1]; a += 32)
      if (take(a)) {
        const int o = poss[a] - pbase;
        atomicOr(&bits[o >> 5], 1u << (o & 31));
      }
    __syncwarp();
    // exclusive scan of the slice counts, lane l holding slices [l*B, l*B + B)
    const int B = (S + 31) >> 5;
    int run = 0;
    for (int b = lane * B; b < S && b < lane * B + B; ++b)
      run += __popc(bits[2 * b]) + __popc(bits[2 * b + 1]);
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    int at = incl - run;
    const int64_t rp = int64_t(r) * N + px_of[r];
    int32_t* orow = kept_off + rp * Sp;
    int2* erow = kept + rp * k;  // the round's entries, from 0
    for (int b = lane * B; b < S && b < lane * B + B; ++b) {
      soff[b] = at;
      orow[b] = at;
      at += __popc(bits[2 * b]) + __popc(bits[2 * b + 1]);
    }
    if (lane == 0) orow[S] = total;
    __syncwarp();
    for (int a = rb[r] + lane; a < rb[r + 1]; a += 32) {
      if (!take(a)) continue;
      const int32_t pos = poss[a];
      const int o = pos - pbase, wi = o >> 5;
      const int dest = soff[o >> 6] + __popc(bits[wi] & ((1u << (o & 31)) - 1u)) +
                       ((wi & 1) ? __popc(bits[wi - 1]) : 0);
      const float sc = key_score(keys[a]);
      srow[ns + dest] = py[int64_t(r) * C + pos];
      uint32_t packed = 0u;
      if (z_ok) {
        const float pr = expf(sc - lse);
        const __nv_bfloat16 h = __float2bfloat16_rn(pr);
        const __nv_bfloat16 l = __float2bfloat16_rn(pr - __bfloat162float(h));
        packed = uint32_t(__bfloat16_as_ushort(h)) | (uint32_t(__bfloat16_as_ushort(l)) << 16);
      }
      erow[dest] = make_int2(pos, int32_t(packed));
      if (lg) lg[1 + ns + dest] = sc;
      worst = fminf(worst, sc);
    }
    ns += total;
    __syncwarp();
  }
  worst = -warp_max(-worst);
  if constexpr (!kGrouped) lse = m + logf(warp_sum(acc) + expf(lp - m));
  for (int a = ns + lane; a < k; a += 32) {
    srow[a] = -1;
    if (lg) lg[1 + a] = -INFINITY;
  }
  if (lane == 0) {
    if (lg) lg[0] = z_ok ? lp : NAN;
    if (kGrouped) pos_logit[i] = z_ok ? lp : NAN;
  }

  // theta_max: the largest score some round did not emit (-inf if every round emitted
  // all); the k-th kept score is the smallest kept one
  const float s_k = ns < k ? -INFINITY : worst;
  if (lane == 0 && (overflow || (theta_max > -INFINITY && theta_max >= s_k))) {
    atomicAdd(status + 1, 1u);
    if (overflow) atomicAdd(status + 2, 1u);
    raise_flag(status, RECE_DEVICE_INEXACT);
  }

  if (lane == 0) {
    if (!z_ok) {
      raise_flag(status, RECE_DEVICE_BAD_TARGET);
      lse_out[i] = NAN;
      if (row_loss) row_loss[i] = NAN;
    } else {
      lse_out[i] = lse;
      if (row_loss) row_loss[i] = lse - lp;
    }
  }
  return true;
}

// Fast path: one row per warp, candidates in shared memory (cap per row).
template <typename T, bool kGrouped, int kGather>
__global__ void __launch_bounds__(kThreads) k_merge_tc(const MergeArgs<T> A, int cap) {
  extern __shared__ __align__(16) uint8_t sh_raw[];
  const int warps = blockDim.x >> 5, wid = threadIdx.x >> 5;
  const size_t tab = merge_table_bytes(kGrouped, A.Sp);
  const size_t per_warp = size_t(cap) * 8 + tab;
  uint8_t* base = sh_raw + per_warp * wid;
  uint32_t* cnt = reinterpret_cast<uint32_t*>(base);
  uint32_t* keys = reinterpret_cast<uint32_t*>(base + tab);
  int32_t* poss = reinterpret_cast<int32_t*>(keys + cap);
  const int64_t i = int64_t(blockIdx.x) * warps + wid;
  if (i >= A.N) return;  // whole warp leaves together; no block-wide barriers follow
  merge_row<T, kGrouped, kGather>(A, i, cnt, keys, poss, cap, true);
}

// Spilled rows: the warps walk the spill list with their candidates in global scratch
// (room for every list entry of every round, so nothing is dropped).
template <typename T, bool kGrouped, int kGather>
__global__ void __launch_bounds__(kThreads) k_merge_tc_spill(const MergeArgs<T> A, int cap,
                                                             uint32_t* scratch) {
  extern __shared__ __align__(16) uint8_t sh_raw[];
  const int wid = threadIdx.x >> 5;
  uint32_t* cnt = reinterpret_cast<uint32_t*>(sh_raw + merge_table_bytes(kGrouped, A.Sp) * wid);
  const int64_t gw = int64_t(blockIdx.x) * (blockDim.x >> 5) + wid;
  const int64_t nw = int64_t(gridDim.x) * (blockDim.x >> 5);
  uint32_t* keys = scratch + gw * 2 * int64_t(cap);
  int32_t* poss = reinterpret_cast<int32_t*>(keys + cap);
  const uint32_t n = *reinterpret_cast<volatile uint32_t*>(A.spill_count);
  for (int64_t w = gw; w < n; w += nw)
    merge_row<T, kGrouped, kGather>(A, A.spill_rows[w], cnt, keys, poss, cap, false);
}

// ---------------------------------------------------------------- one row per CTA
// The same merge with the row's work spread over four warps: warp w reads sub-list w of
// every round (the entries of selection warpgroup w) into its own shared-memory region,
// the k-th key is found with 8-bit digits over a shared 256-bin histogram, and in grouped
// mode the kept entries of a round go out ordered by sorted position (a bit map of the
// round's window: an entry's place is the count of kept positions before it), which
// groups them by 64-position slice with no sort.  Without grouping they go out by round,
// then warp, lane and place in the region.  Every sum is taken in a fixed order.  A row
// whose entries do not fit a warp's region is handed to the spill list (the warp-per-row
// path above finishes it).
constexpr int kCtaThreads = 128;
constexpr int kCtaWarps = kCtaThreads / 32;
constexpr int kGatherCta = 4;  // list entries per lane in flight

struct CtaShared {
  uint32_t u[kCtaWarps][3];  // per warp: or, and, largest of its keys
  int cnt[kCtaWarps];        // per warp: entries that passed (uncapped)
  int rb[kCtaWarps][9];      // per warp: where each round's entries start in its region
  float f[kCtaWarps][3];     // per warp: positive-logit part, sum of exponentials, worst
  int scan[kCtaWarps];       // warp totals of a block scan
  int res[3];                // selection pass: digit, keys above it, keys in it
  int px[8], cx[8];          // the row's sorted position and chunk, per round
};

struct CtaSel {
  uint32_t T;
  int need;
  int eq;
};

// Exclusive scan of v over the block (thread order); total gets the sum.  Starts and ends
// with every thread past a barrier, so cs.scan may be reused right after.
__device__ __forceinline__ int cta_excl_scan(int v, CtaShared& cs, int& total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) cs.scan[wid] = incl;
  __syncthreads();
  int base = 0, all = 0;
#pragma unroll
  for (int w = 0; w < kCtaWarps; ++w) {
    base += w < wid ? cs.scan[w] : 0;
    all += cs.scan[w];
  }
  total = all;
  __syncthreads();
  return base + incl - v;
}

// The want-th largest (1-based) of the keys in play over the four warps' regions
// (get(q, key) -> in play, its key; q < nq in this warp's region); orv / andv / m: the OR,
// AND and count of those keys.  Digits of 8 bits from the highest bit in which the keys
// differ; same result convention as warp_select_kth.
template <typename Get>
__device__ CtaSel cta_select_kth(int nq, int want, uint32_t orv, uint32_t andv, int m, Get get,
                                 uint32_t* hist, CtaShared& cs) {
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t diff = orv ^ andv;
  if (diff == 0u) return CtaSel{andv, want, m};
  const int hb = 31 - __clz(diff);
  int shift = hb >= 7 ? hb - 7 : 0;
  uint32_t pmask = shift + 8 >= 32 ? 0u : ~((1u << (shift + 8)) - 1u);
  uint32_t prefix = andv & pmask;
  for (;;) {
    hist[tid] = 0u;
    hist[tid + kCtaThreads] = 0u;
    __syncthreads();
    for (int q = lane; q < nq; q += 32) {
      uint32_t key;
      if (get(q, key) && (key & pmask) == prefix)
        atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    // thread t: digits 255 - 2t and 254 - 2t, i.e. the digits in descending order
    const int c0 = int(hist[255 - 2 * tid]), c1 = int(hist[254 - 2 * tid]);
    int total;
    const int excl = cta_excl_scan(c0 + c1, cs, total);
    if (excl < want && want <= excl + c0) {
      cs.res[0] = 255 - 2 * tid;
      cs.res[1] = excl;
      cs.res[2] = c0;
    } else if (excl + c0 < want && want <= excl + c0 + c1) {
      cs.res[0] = 254 - 2 * tid;
      cs.res[1] = excl + c0;
      cs.res[2] = c1;
    }
    __syncthreads();
    const int dg = cs.res[0], above = cs.res[1], count = cs.res[2];
    want -= above;
    // (a digit below 8 bits wide at the bottom overlaps bits the prefix already fixed;
    // every key counted agrees with the prefix there, so the OR changes nothing there)
    prefix |= uint32_t(dg) << shift;
    pmask |= 255u << shift;
    if (count == want || shift == 0) return CtaSel{prefix, want, count};
    shift = shift >= 8 ? shift - 8 : 0;
  }
}

template <typename T, bool kGrouped>
__global__ void __launch_bounds__(kCtaThreads, 8) k_merge_cta(const MergeArgs<T> A, int capw) {
  extern __shared__ __align__(16) uint8_t sh_raw[];
  __shared__ CtaShared cs;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int64_t i = blockIdx.x;
  const int64_t N = A.N, C = A.C;
  const int k = A.k, n_r = A.n_r, n_c = A.n_c, n_ec = A.n_ec, Qw = A.Qw, Sp = A.Sp;
  const int32_t* __restrict__ py = A.py;
  const int32_t* __restrict__ invX = A.invX;
  uint32_t* keys = reinterpret_cast<uint32_t*>(sh_raw) + size_t(wid) * 2 * capw;
  int32_t* poss = reinterpret_cast<int32_t*>(keys + capw);
  uint32_t* aux = reinterpret_cast<uint32_t*>(sh_raw) + size_t(kCtaWarps) * 2 * capw;
  const int aux_words = kGrouped && 2 * Sp > 256 ? 2 * Sp : 256;
  int32_t* sliceoff = reinterpret_cast<int32_t*>(aux + aux_words);

  const int32_t z = A.targets[i];
  const bool z_ok = z >= 0 && z < C;
  // the row's sorted position and chunk in each round
  if (tid < n_r) {
    const int px = invX[int64_t(tid) * N + i];
    cs.px[tid] = px;
    cs.cx[tid] = int((int64_t(px) * n_c) / N);
  }
  __syncthreads();

  // 1. this warp's sub-list of every round: entries above the round's theta, not the
  //    positive, not in an earlier round's window; their keys and sorted positions
  int n = 0;
  uint32_t orv = 0u, andv = 0xFFFFFFFFu, kmax = 0u;
  bool over = false;
  float theta_max = -INFINITY;
  for (int r = 0; r < n_r; ++r) {
    if (lane == 0) cs.rb[wid][r] = n < capw ? n : capw;
    const int64_t rp = int64_t(r) * N + cs.px[r];
    const int4 c4 = A.list_count[rp];
    const float th = A.list_theta[rp];
    theta_max = fmaxf(theta_max, th);
    over |= c4.x > Qw || c4.y > Qw || c4.z > Qw || c4.w > Qw;
    const int cw0 = wid == 0 ? c4.x : wid == 1 ? c4.y : wid == 2 ? c4.z : c4.w;
    const int cw = cw0 < Qw ? cw0 : Qw;
    const int32_t pz = z_ok ? A.invY[int64_t(r) * C + z] : -1;
    const int2* L = A.list + (rp * 4 + wid) * Qw;
    for (int a0 = 0; a0 < cw; a0 += 32 * kGatherCta) {
      int2 e[kGatherCta];
      bool keep[kGatherCta];
#pragma unroll
      for (int u = 0; u < kGatherCta; ++u) {
        const int a = a0 + 32 * u + lane;
        e[u] = a < cw ? L[a] : make_int2(0, 0);
        keep[u] = a < cw && __int_as_float(e[u].x) > th && e[u].y != pz;
      }
      if (r > 0) {  // an item an earlier round's window held was that round's to select
#pragma unroll
        for (int u = 0; u < kGatherCta; ++u) {
          const int32_t jj = keep[u] ? py[int64_t(r) * C + e[u].y] : 0;
          for (int q = 0; q < r && keep[u]; ++q) {
            const int dc = A.chunkY[int64_t(q) * C + jj] - cs.cx[q];
            if (dc >= -n_ec && dc <= n_ec) keep[u] = false;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kGatherCta; ++u) {
        const unsigned b = __ballot_sync(0xFFFFFFFFu, keep[u]);
        if (keep[u]) {
          const int at = n + __popc(b & ((1u << lane) - 1u));
          const uint32_t key = score_key(__int_as_float(e[u].x));
          if (at < capw) {
            keys[at] = key;
            poss[at] = e[u].y;
          }
          orv |= key;
          andv &= key;
          kmax = key > kmax ? key : kmax;
        }
        n += __popc(b);
      }
    }
  }
  // the positive's logit, over the block
  float part = 0.0f;
  if (z_ok) {
    const T* x = A.X + i * A.d;
    const T* y = A.Y + int64_t(z) * A.d;
    for (int t = tid; t < A.d; t += kCtaThreads) part = fmaf(to_f32(x[t]), to_f32(y[t]), part);
  }
  part = warp_sum(part);
  orv = warp_or(orv);
  andv = warp_and(andv);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint32_t v = __shfl_xor_sync(0xFFFFFFFFu, kmax, o);
    kmax = v > kmax ? v : kmax;
  }
  if (lane == 0) {
    cs.rb[wid][n_r] = n < capw ? n : capw;
    cs.cnt[wid] = n;
    cs.u[wid][0] = orv;
    cs.u[wid][1] = andv;
    cs.u[wid][2] = kmax;
    cs.f[wid][0] = part;
  }
  __syncthreads();
  int ntot = 0;
  bool spill = false;
  float lp = 0.0f;
  orv = 0u;
  andv = 0xFFFFFFFFu;
  kmax = 0u;
#pragma unroll
  for (int w = 0; w < kCtaWarps; ++w) {
    ntot += cs.cnt[w];
    spill |= cs.cnt[w] > capw;
    lp += cs.f[w][0];
    if (cs.cnt[w] > 0) {
      orv |= cs.u[w][0];
      andv &= cs.u[w][1];
      kmax = cs.u[w][2] > kmax ? cs.u[w][2] : kmax;
    }
  }
  if (spill) {  // (the whole block leaves)
    if (tid == 0) A.spill_rows[atomicAdd(A.spill_count, 1u)] = int32_t(i);
    return;
  }
  const int* rbw = cs.rb[wid];  // (not written again)
  const int nq = rbw[n_r];
  auto item_of = [&](int q) {
    int r = 0;
    while (r + 1 < n_r && q >= rbw[r + 1]) ++r;
    return py[int64_t(r) * C + poss[q]];
  };

  // 2. the k best
  const int kk = k < ntot ? k : ntot;
  const bool all = kk >= ntot;
  CtaSel s1{0u, 0, 0}, s2{0u, 0, 0};
  bool tie = false;
  if (!all) {
    s1 = cta_select_kth(
        nq, kk, orv, andv, ntot, [&](int q, uint32_t& key) { key = keys[q]; return true; }, aux,
        cs);
    if (s1.need != s1.eq) {
      tie = true;
      const uint32_t Tk = s1.T;
      uint32_t o2 = 0u, a2 = 0xFFFFFFFFu;
      int m2 = 0;
      for (int q = lane; q < nq; q += 32)
        if (keys[q] == Tk) {
          const uint32_t v = ~uint32_t(item_of(q));
          o2 |= v;
          a2 &= v;
          ++m2;
        }
      o2 = warp_or(o2);
      a2 = warp_and(a2);
      m2 = int(warp_sum(float(m2)));
      __syncthreads();  // cs.u was read above by every thread
      if (lane == 0) {
        cs.u[wid][0] = o2;
        cs.u[wid][1] = a2;
        cs.cnt[wid] = m2;
      }
      __syncthreads();
      o2 = 0u;
      a2 = 0xFFFFFFFFu;
      m2 = 0;
#pragma unroll
      for (int w = 0; w < kCtaWarps; ++w) {
        m2 += cs.cnt[w];
        if (cs.cnt[w] > 0) {
          o2 |= cs.u[w][0];
          a2 &= cs.u[w][1];
        }
      }
      s2 = cta_select_kth(
          nq, s1.need, o2, a2, m2,
          [&](int q, uint32_t& key) {
            if (keys[q] != Tk) return false;
            key = ~uint32_t(item_of(q));
            return true;
          },
          aux, cs);
    }
  }
  auto take = [&](int q) {
    const uint32_t key = keys[q];
    return all || key > s1.T || (key == s1.T && (!tie || ~uint32_t(item_of(q)) >= s2.T));
  };

  // 3. the row's loss (RECE, Algorithm 1's loss lines); the best candidate is always kept
  const float best = ntot > 0 ? key_score(kmax) : -INFINITY;
  const float m = fmaxf(lp, best);
  float acc = 0.0f, worst = INFINITY;
  for (int q = lane; q < nq; q += 32)
    if (take(q)) {
      const float sc = key_score(keys[q]);
      acc += expf(sc - m);
      worst = fminf(worst, sc);
    }
  acc = warp_sum(acc);
  worst = warp_max(-worst);
  if (lane == 0) {
    cs.f[wid][1] = acc;
    cs.f[wid][2] = worst;
  }
  __syncthreads();
  float sum = 0.0f;
  worst = INFINITY;
#pragma unroll
  for (int w = 0; w < kCtaWarps; ++w) {
    sum += cs.f[w][1];
    worst = fminf(worst, -cs.f[w][2]);
  }
  const float lse = m + logf(sum + expf(lp - m));

  // 4. the kept entries, round by round
  float* lg = A.logits ? A.logits + i * (int64_t(k) + 1) : nullptr;
  int32_t* srow = A.selected + i * k;
  int ns = 0;
  for (int r = 0; r < n_r; ++r) {
    const int px = cs.px[r];
    if constexpr (kGrouped) {
      // ordered by sorted position: a bit per position of the round's window, from the
      // start of its first 64-position slice
      const int64_t c = cs.cx[r];
      const int64_t w0 = chunk_start(c - n_ec < 0 ? 0 : c - n_ec, C, n_c);
      const int64_t w1 = chunk_start(c + n_ec + 1 > n_c ? n_c : c + n_ec + 1, C, n_c);
      const int sig0 = int(w0 >> 6);
      const int S = w1 > w0 ? int((w1 - 1) >> 6) - sig0 + 1 : 0;
      const int32_t base = sig0 << 6;
      uint32_t* bits = aux;
      for (int b = tid; b < 2 * S; b += kCtaThreads) bits[b] = 0u;
      __syncthreads();
      for (int q = rbw[r] + lane; q < rbw[r + 1]; q += 32)
        if (take(q)) {
          const int o = poss[q] - base;
          atomicOr(&bits[o >> 5], 1u << (o & 31));
        }
      __syncthreads();
      // slices [t*B, t*B + B) per thread: counts, then their starts
      const int B = (S + kCtaThreads - 1) / kCtaThreads;
      const int s0 = tid * B, s1e = s0 + B < S ? s0 + B : S;
      int run = 0;
      for (int s = s0; s < s1e; ++s) run += __popc(bits[2 * s]) + __popc(bits[2 * s + 1]);
      int total;
      int at = cta_excl_scan(run, cs, total);
      const int64_t rp = int64_t(r) * N + px;
      int32_t* orow = A.kept_off + rp * Sp;
      for (int s = s0; s < s1e; ++s) {
        sliceoff[s] = at;
        orow[s] = at;
        at += __popc(bits[2 * s]) + __popc(bits[2 * s + 1]);
      }
      if (tid == 0) orow[S] = total;
      __syncthreads();
      int2* erow = A.kept + rp * k;
      for (int q = rbw[r] + lane; q < rbw[r + 1]; q += 32) {
        if (!take(q)) continue;
        const int32_t pos = poss[q];
        const int o = pos - base, wi = o >> 5;
        const int dest = sliceoff[o >> 6] + __popc(bits[wi] & ((1u << (o & 31)) - 1u)) +
                         ((wi & 1) ? __popc(bits[wi - 1]) : 0);
        const float sc = key_score(keys[q]);
        uint32_t packed = 0u;
        if (z_ok) {
          const float pr = expf(sc - lse);
          const __nv_bfloat16 h = __float2bfloat16_rn(pr);
          const __nv_bfloat16 l = __float2bfloat16_rn(pr - __bfloat162float(h));
          packed = uint32_t(__bfloat16_as_ushort(h)) | (uint32_t(__bfloat16_as_ushort(l)) << 16);
        }
        erow[dest] = make_int2(pos, int32_t(packed));
        srow[ns + dest] = py[int64_t(r) * C + pos];
        if (lg) lg[1 + ns + dest] = sc;
      }
      ns += total;
      __syncthreads();  // the bit map is cleared again by the next round
    } else {
      int mine = 0;
      for (int q = rbw[r] + lane; q < rbw[r + 1]; q += 32) mine += take(q) ? 1 : 0;
      int total;
      int at = ns + cta_excl_scan(mine, cs, total);
      for (int q = rbw[r] + lane; q < rbw[r + 1]; q += 32) {
        if (!take(q)) continue;
        const float sc = key_score(keys[q]);
        srow[at] = py[int64_t(r) * C + poss[q]];
        if (lg) lg[1 + at] = sc;
        ++at;
      }
      ns += total;
    }
  }
  for (int a = ns + tid; a < k; a += kCtaThreads) {
    srow[a] = -1;
    if (lg) lg[1 + a] = -INFINITY;
  }
  if (tid == 0) {
    if (lg) lg[0] = z_ok ? lp : NAN;
    if (kGrouped) A.pos_logit[i] = z_ok ? lp : NAN;
    // exactness: theta_max is the largest score some round did not emit
    const float s_k = ns < k ? -INFINITY : worst;
    if (over || (theta_max > -INFINITY && theta_max >= s_k)) {
      atomicAdd(A.status + 1, 1u);
      if (over) atomicAdd(A.status + 2, 1u);
      raise_flag(A.status, RECE_DEVICE_INEXACT);
    }
    if (!z_ok) {
      raise_flag(A.status, RECE_DEVICE_BAD_TARGET);
      A.lse_out[i] = NAN;
      if (A.row_loss) A.row_loss[i] = NAN;
    } else {
      A.lse_out[i] = lse;
      if (A.row_loss) A.row_loss[i] = lse - lp;
    }
  }
}

}  // namespace

int tc_list_capacity(int k);

// Candidates buffered per row in shared memory: a round emits about k + 1 + (one histogram
// bin) entries, so k + k/4 + 64 per round holds nearly every row; the few that bring more
// go to the spill path.
int merge_tc_cap(int n_r, int k) { return n_r * (k + k / 4 + 64); }
// The spill path's buffer: every list entry of every round.
int merge_tc_spill_cap(int n_r, int k) { return n_r * tc_list_capacity(k); }
constexpr int kSpillWarps = 1024;
size_t merge_tc_spill_bytes(int n_r, int k) {
  return size_t(kSpillWarps) * size_t(merge_tc_spill_cap(n_r, k)) * 8;
}

// (the largest table: grouped, the widest window the plan accepts)
size_t merge_tc_warp_bytes(int n_r, int k) {
  return size_t(merge_tc_cap(n_r, k)) * 8 + merge_table_bytes(true, kMaxKeptSlices + 1);
}

// One-row-per-CTA path: the 256-bin histogram, which the grouped output's bit map (two
// words per slice) reuses, and the slice starts; then each warp's region for the entries
// of its sub-lists that pass, as large as eight CTAs per SM allow (the registers allow
// eight), but never more than the sub-lists can hold.  The path is taken when k >= 512
// (smaller rows are done faster a warp each, more rows in flight) and the region holds at
// least a quarter of the warp path's buffer plus 32 (the sub-lists hold every fourth tile
// of the window, so their shares stay close to a quarter).
constexpr size_t kCtaSmemBudget = 26 * 1024;
size_t merge_cta_aux_bytes(int Sp) {
  const size_t aux = 2 * size_t(Sp) > 256 ? 2 * size_t(Sp) : 256;
  return aux * 4 + size_t(Sp) * 4;
}
int merge_cta_region(int n_r, int k, int Sp) {
  const size_t aux = merge_cta_aux_bytes(Sp);
  if (aux >= kCtaSmemBudget) return 0;
  const int64_t fit = int64_t((kCtaSmemBudget - aux) / (size_t(kCtaWarps) * 8));
  const int64_t most = int64_t(n_r) * tc_sublist_capacity(k);
  const int64_t want = int64_t(n_r) * ((k + k / 4 + 64 + 3) / 4) + 32;
  if (k < 512 || fit < want) return 0;
  return int(fit < most ? fit : most);
}
size_t merge_cta_smem(int capw, int Sp) {
  return size_t(kCtaWarps) * 8 * size_t(capw) + merge_cta_aux_bytes(Sp);
}

template <typename T>
cudaError_t launch_merge_tc(const rece_plan_s& p, const T* X, const T* Y, const int32_t* targets,
                            const int32_t* py, const int32_t* invX, const int32_t* invY,
                            const int32_t* chunkY, const int2* list, const int4* list_count,
                            const float* list_theta, int32_t* selected, int2* kept,
                            int32_t* kept_off, float* pos_logit, int Sp, float* lse,
                            float* row_loss, float* logits, uint32_t* status, int32_t* spill_rows,
                            void* spill_scratch, cudaStream_t st) {
  const auto& c = p.cfg;
  if (c.N == 0) return cudaSuccess;
  MergeArgs<T> A{};
  A.X = X;
  A.Y = Y;
  A.targets = targets;
  A.py = py;
  A.invX = invX;
  A.invY = invY;
  A.chunkY = chunkY;
  A.list = list;
  A.list_count = list_count;
  A.list_theta = list_theta;
  A.N = c.N;
  A.C = c.C;
  A.d = c.d;
  A.k = c.k;
  A.n_r = c.n_r;
  A.n_c = c.n_c;
  A.n_ec = c.n_ec;
  A.Qw = tc_sublist_capacity(c.k);
  A.Sp = Sp;
  A.selected = selected;
  A.kept = kept;
  A.kept_off = kept_off;
  A.pos_logit = pos_logit;
  A.lse_out = lse;
  A.row_loss = row_loss;
  A.logits = logits;
  A.status = status;
  A.spill_rows = spill_rows;
  A.spill_count = status + 3;
  const bool grouped = kept != nullptr;
  const bool wide = c.k >= 384;
  cudaError_t e = cudaMemsetAsync(A.spill_count, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  const int capw = merge_cta_region(c.n_r, c.k, grouped ? Sp : 0);
  const size_t cta_smem = merge_cta_smem(capw, grouped ? Sp : 0);
  if (invY && capw > 0) {
    auto kern = grouped ? k_merge_cta<T, true> : k_merge_cta<T, false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(cta_smem));
    if (e != cudaSuccess) return e;
    kern<<<unsigned(c.N), kCtaThreads, cta_smem, st>>>(A, capw);
  } else {
    const int cap = merge_tc_cap(c.n_r, c.k);
    const size_t per_warp = size_t(cap) * 8 + merge_table_bytes(grouped, Sp);
    int warps = int((200 * 1024) / per_warp);
    warps = warps < 1 ? 1 : (warps > kThreads / 32 ? kThreads / 32 : warps);
    const size_t smem = per_warp * warps;
    auto kern = grouped ? (wide ? k_merge_tc<T, true, 8> : k_merge_tc<T, true, 4>)
                        : (wide ? k_merge_tc<T, false, 8> : k_merge_tc<T, false, 4>);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    kern<<<unsigned(ceil_div(c.N, warps)), warps * 32, smem, st>>>(A, cap);
  }
  auto spill = grouped ? (wide ? k_merge_tc_spill<T, true, 8> : k_merge_tc_spill<T, true, 4>)
                       : (wide ? k_merge_tc_spill<T, false, 8> : k_merge_tc_spill<T, false, 4>);
  const size_t spill_smem = size_t(kThreads / 32) * merge_table_bytes(grouped, Sp);
  e = cudaFuncSetAttribute(spill, cudaFuncAttributeMaxDynamicSharedMemorySize, int(spill_smem));
  if (e != cudaSuccess) return e;
  spill<<<kSpillWarps / (kThreads / 32), kThreads, spill_smem, st>>>(
      A, merge_tc_spill_cap(c.n_r, c.k), static_cast<uint32_t*>(spill_scratch));
  count_launches(2);
  return cudaGetLastError();
}

template cudaError_t launch_merge_tc<__nv_bfloat16>(
    const rece_plan_s&, const __nv_bfloat16*, const __nv_bfloat16*, const int32_t*,
    const int32_t*, const int32_t*, const int32_t*, const int32_t*, const int2*, const int4*,
    const float*,
    int32_t*, int2*, int32_t*, float*, int, float*, float*, float*, uint32_t*, int32_t*, void*,
    cudaStream_t);

}  // namespace rece
