// merge_tc.cu -- steps 4-5 for the tensor-core selection: one warp per row.
//
// The row's candidates are the (score, sorted position) pairs its rounds emitted.  A pair
// of round r is translated to its item j and dropped when j is the row's positive or when
// j also lies in the row's window of an earlier round r' < r (that round saw the same
// pair, so the union of the rounds stays de-duplicated -- the RECE paper's ln(count)
// correction for repeated pairs amounts to counting each pair once).  The k best of the
// rest by (score descending, item ascending) are found with a warp radix select (4-bit
// digits of the score key from its highest varying bit, then the item ids if the k-th
// place is tied), kept in the order of the candidate lists (a fixed order), and give the
// row's loss (RECE, Algorithm 1's loss lines):
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
  // The kept entries, by round and, within a round, grouped by 64-position slice of the
  // round's sorted catalogue (in candidate-list order inside a slice): a stable counting
  // sort over the slices of the row's window.  Besides the row's outputs (items, logits),
  // the backward gets, indexed by (round, sorted row p): the round's entries
  // kept[r][p][e] = (sorted position, p_ij as two bf16 halves hi | lo << 16, with
  // p_ij = exp(l_ij - lse_i) = bf16(hi) + bf16(lo) to about 16 bits; 0 for a bad target)
  // and the slice starts kept_off[r][p][s] (s = 0..S, entry S = the round's count).
  float* lg = logits ? logits + i * (int64_t(k) + 1) : nullptr;
  int32_t* srow = selected + i * k;
  int32_t* bins = reinterpret_cast<int32_t*>(cnt);  // up to 512 slices (the count table)
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
    for (int b = lane; b < S; b += 32) bins[b] = 0;
    __syncwarp();
    for (int a = rb[r] + lane; a < rb[r + 1]; a += 32)
      if (take(a)) atomicAdd(&bins[(poss[a] >> 6) - sig0], 1);
    __syncwarp();
    // exclusive scan of the slice counts, lane l holding slices [l*B, l*B + B)
    const int B = (S + 31) >> 5;
    int sbits = 0;  // bits of the slice ids 0..S-1
    while ((1 << sbits) < S) ++sbits;
    int run = 0;
    for (int b = lane * B; b < S && b < lane * B + B; ++b) run += bins[b];
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    int at = ns + incl - run;
    const int64_t rp = int64_t(r) * N + px_of[r];
    int32_t* orow = kept_off + rp * Sp;
    int2* erow = kept + rp * k;  // the round's entries, from 0
    for (int b = lane * B; b < S && b < lane * B + B; ++b) {
      const int v = bins[b];
      bins[b] = at;
      orow[b] = at - ns;
      at += v;
    }
    if (lane == 0) orow[S] = total;
    __syncwarp();
    for (int a0 = rb[r]; a0 < rb[r + 1]; a0 += 32) {
      const int a = a0 + lane;
      const bool tk = a < rb[r + 1] && take(a);
      const int sl = tk ? (poss[a] >> 6) - sig0 : 0;
      const unsigned peers = digit_peers(sl, sbits, tk, lane);
      const int dest = tk ? bins[sl] + __popc(peers & ((1u << lane) - 1u)) : 0;
      __syncwarp();
      if (tk && lane == __ffs(peers) - 1) bins[sl] += __popc(peers);
      __syncwarp();
      if (tk) {
        const int32_t pos = poss[a];
        const float sc = key_score(keys[a]);
        srow[dest] = py[int64_t(r) * C + pos];
        uint32_t packed = 0u;
        if (z_ok) {
          const float pr = expf(sc - lse);
          const __nv_bfloat16 h = __float2bfloat16_rn(pr);
          const __nv_bfloat16 l = __float2bfloat16_rn(pr - __bfloat162float(h));
          packed = uint32_t(__bfloat16_as_ushort(h)) | (uint32_t(__bfloat16_as_ushort(l)) << 16);
        }
        erow[dest - ns] = make_int2(pos, int32_t(packed));
        if (lg) lg[1 + dest] = sc;
        worst = fminf(worst, sc);
      }
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
  const size_t per_warp = size_t(cap) * 8 + kCountBytes;
  uint8_t* base = sh_raw + per_warp * wid;
  uint32_t* cnt = reinterpret_cast<uint32_t*>(base);
  uint32_t* keys = reinterpret_cast<uint32_t*>(base + kCountBytes);
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
  __shared__ uint32_t sh_cnt[kThreads / 32][kCountBytes / 4];
  const int wid = threadIdx.x >> 5;
  const int64_t gw = int64_t(blockIdx.x) * (blockDim.x >> 5) + wid;
  const int64_t nw = int64_t(gridDim.x) * (blockDim.x >> 5);
  uint32_t* keys = scratch + gw * 2 * int64_t(cap);
  int32_t* poss = reinterpret_cast<int32_t*>(keys + cap);
  const uint32_t n = *reinterpret_cast<volatile uint32_t*>(A.spill_count);
  for (int64_t w = gw; w < n; w += nw)
    merge_row<T, kGrouped, kGather>(A, A.spill_rows[w], sh_cnt[wid], keys, poss, cap, false);
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

size_t merge_tc_warp_bytes(int n_r, int k) {
  return size_t(merge_tc_cap(n_r, k)) * 8 + kCountBytes;
}

template <typename T>
cudaError_t launch_merge_tc(const rece_plan_s& p, const T* X, const T* Y, const int32_t* targets,
                            const int32_t* py, const int32_t* invX, const int32_t* chunkY,
                            const int2* list, const int4* list_count,
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
  const int cap = merge_tc_cap(c.n_r, c.k);
  const size_t per_warp = merge_tc_warp_bytes(c.n_r, c.k);
  int warps = int((200 * 1024) / per_warp);
  warps = warps < 1 ? 1 : (warps > kThreads / 32 ? kThreads / 32 : warps);
  const size_t smem = per_warp * warps;
  const bool grouped = kept != nullptr;
  const bool wide = c.k >= 384;
  auto kern = grouped ? (wide ? k_merge_tc<T, true, 8> : k_merge_tc<T, true, 4>)
                      : (wide ? k_merge_tc<T, false, 8> : k_merge_tc<T, false, 4>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(A.spill_count, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  kern<<<unsigned(ceil_div(c.N, warps)), warps * 32, smem, st>>>(A, cap);
  auto spill = grouped ? (wide ? k_merge_tc_spill<T, true, 8> : k_merge_tc_spill<T, true, 4>)
                       : (wide ? k_merge_tc_spill<T, false, 8> : k_merge_tc_spill<T, false, 4>);
  spill<<<kSpillWarps / (kThreads / 32), kThreads, 0, st>>>(
      A, merge_tc_spill_cap(c.n_r, c.k), static_cast<uint32_t*>(spill_scratch));
  count_launches(2);
  return cudaGetLastError();
}

template cudaError_t launch_merge_tc<__nv_bfloat16>(
    const rece_plan_s&, const __nv_bfloat16*, const __nv_bfloat16*, const int32_t*,
    const int32_t*, const int32_t*, const int32_t*, const int2*, const int4*, const float*,
    int32_t*, int2*, int32_t*, float*, int, float*, float*, float*, uint32_t*, int32_t*, void*,
    cudaStream_t);

}  // namespace rece
