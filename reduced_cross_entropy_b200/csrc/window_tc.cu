// window_tc.cu -- the all-negatives mode on the tcgen05 tensor cores (bf16, d <= 256):
// Algorithm 1 of the RECE paper as printed (section 3), every item of a row's chunk window
// a negative, over n_r rounds with the rounds paragraph's duplicate correction (a pair
// computed in cnt of the rounds enters each round's sum as exp(l - ln cnt) = exp(l)/cnt).
// The positive is left out of the window sums (it enters once, as l+).
//
// One kernel, three roles, all on the dense band of a round: sorted rows of chunk c
// against the sorted catalogue positions of chunks c-n_ec..c+n_ec.  A work item is 128
// consecutive sorted positions of the M side and streams the union of their windows (K
// side) in 128-wide tiles; every tile's scores S = A B^T (K = d) are formed in TMEM.
//   LSE  M = rows, K = items.  Each row's thread keeps an online (max, sum) of
//        exp(s) / cnt over its window columns; out: the round's (max, sum) per row.
//   DX   M = rows, K = items.  P = exp(s - lse_row) / cnt on the row's window columns,
//        O += P V with V = the K tile of the sorted catalogue copy (read MN-major); at the end
//        dX[row] += O * dloss / N.
//   DY   M = items, K = rows.  The same with the roles swapped (the pair is live when the
//        item lies in the row's window), V = the sorted copy of X; dY[item] +=.
// The round count of a pair (row p, item q) is 1 plus the number of other rounds s in
// which the item's chunk is within n_ec of the row's chunk: both come from per-round
// tables of every row's and item's chunk in every round.
//
// Warps: 0 TMA producer, 1 MMA issuer, 2-17 epilogue (warpgroup g takes columns
// 32g..32g+31 of each score tile; warp w reads TMEM lanes 32 (w % 4)..).  TMEM: two score
// buffers of 128 columns (the MMA forms tile t+1 while the epilogue reads tile t) and, in
// the gradient roles, the 128 x d accumulator O.  P goes to shared memory split as
// hi + lo bf16 (hi = bf16(p), lo = bf16(p - hi)) in the 128-byte-swizzled K-major layout;
// both halves are multiplied, so about 16 bits of p reach the products.
//
// Determinism: each output row gets one read-modify-write per launch from the one CTA
// that owns its M tile, K in a fixed order; the positives are written first and the
// rounds add in round order, one launch each.
#include "common.cuh"
#include "plan.h"
#include "sm100.cuh"
#include "tc.h"

namespace rece {
namespace {

using namespace sm100;

constexpr int kRoleLse = 0, kRoleDx = 1, kRoleDy = 2;
constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kBK = 64;
constexpr int kAB = 2;                       // stages of the score operands
constexpr int kEpiWarps = 16;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = 64 + kEpiThreads;
constexpr uint32_t kSlab = kBM * kBK * 2;    // one 128 x 64 bf16 box: 16 KB
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr int kMaxRounds = 8;
constexpr int kMetaPer = ((kMaxRounds + 2) * 128 + 511) / 512;  // metadata loads per thread

struct Ctl {
  uint64_t ab_full[kAB], ab_empty[kAB];
  uint64_t s_full[2], s_empty[2];
  uint64_t v_full[2], v_empty[2];
  uint64_t p_full, p_empty;
  uint64_t done;
  uint32_t tmem_base;
  int abort;
  float part_m[4][kBM], part_s[4][kBM];  // LSE: the warpgroups' partial (max, sum)
  int32_t meta[2][(kMaxRounds + 2) * kBN];  // column metadata of two K tiles
};

// Dynamic shared memory: AB stages, then (gradient roles) V stages and the P tiles.
__host__ __device__ constexpr size_t v_bytes(int d) { return size_t(d) * 256; }  // 2 atoms
__host__ __device__ constexpr size_t window_smem(int role, int d, int nv) {
  return 1024 + size_t(kAB) * 2 * kSlab +
         (role == kRoleLse ? size_t(0) : size_t(nv) * v_bytes(d) + 4 * size_t(kSlab)) +
         sizeof(Ctl);
}

struct Args {
  int64_t N, C;
  int d, n_c, n_ec, n_r, r, nv;
  const int32_t* itemc;      // [n_r][n_r][C]: chunk in round s of the item at sorted q of r
  const int32_t* rowc;       // [n_r][n_r][N]: the same for the rows
  const int32_t* pz;         // [n_r][N]: sorted position of the row's positive (-1: none)
  const float* lse_sorted;   // [n_r][N]
  const int32_t* perm;       // px (DX) or py (DY): sorted position -> row / item
  const float* dloss;
  float* out;                // dX [N][d] or dY [C][d], added into
  float* scratch;            // DX with all rounds in one grid: [n_r][N][d], written
  float2* ms;                // LSE: [n_r][N] (max, sum) of the window terms
  uint32_t* status;
};

__device__ __forceinline__ void on_timeout(Ctl& c, uint32_t* status) {
  *reinterpret_cast<volatile int*>(&c.abort) = 1;
  raise_flag(status, RECE_DEVICE_TIMEOUT);
}

__device__ __forceinline__ int64_t chunk_of(int64_t p, int64_t M, int n_c) {
  return (p * n_c) / M;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Byte offset of 16-byte chunk `ch` (8 bf16) of row `row` in a 128 x 64 swizzled tile.
__device__ __forceinline__ uint32_t sw128_chunk(int row, int ch) {
  return uint32_t((row >> 3) * 1024 + (row & 7) * 128 + (((ch ^ row) & 7) << 4));
}

// 2^x (the hardware approximation; subnormal results flush to zero).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
constexpr float kLog2e = 1.4426950408889634f;

// The K range of an M tile: the union of the windows of its 128 positions, as a start
// rounded down to 64 and a count of 128-wide tiles.
template <int kRole>
__device__ __forceinline__ void k_range(const Args& a, int64_t m0, int64_t& k0a, int& nK) {
  const int64_t Mside = kRole == kRoleDy ? a.C : a.N;
  const int64_t Kside = kRole == kRoleDy ? a.N : a.C;
  const int64_t last = m0 + kBM - 1 < Mside - 1 ? m0 + kBM - 1 : Mside - 1;
  const int64_t cf = chunk_of(m0, Mside, a.n_c), cl = chunk_of(last, Mside, a.n_c);
  const int64_t k0 = chunk_start(cf - a.n_ec < 0 ? 0 : cf - a.n_ec, Kside, a.n_c);
  const int64_t k1 =
      chunk_start(cl + a.n_ec + 1 > a.n_c ? a.n_c : cl + a.n_ec + 1, Kside, a.n_c);
  k0a = k0 & ~int64_t(63);
  nK = k1 > k0 ? int((k1 - k0a + kBN - 1) / kBN) : 0;
}

// kR: the round count the kernel is specialised for (1 or 2), 0 for any up to kMaxRounds.
template <int kRole, int kR>
__global__ void __launch_bounds__(kThreads, 1) k_window_tc(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
    const __grid_constant__ CUtensorMap tmV, const Args a) {
  constexpr bool kGrad = kRole != kRoleLse;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* ab = base;                                    // [kAB][A slab | B slab]
  uint8_t* vbuf = ab + size_t(kAB) * 2 * kSlab;          // [nv][2 atoms of d x 64]
  uint8_t* phi = vbuf + (kGrad ? size_t(a.nv) * v_bytes(a.d) : 0);  // 2 atoms
  uint8_t* plo = phi + (kGrad ? 2 * kSlab : 0);                      // 2 atoms
  Ctl& ctl = *reinterpret_cast<Ctl*>(plo + (kGrad ? 2 * kSlab : 0));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = a.d, nk = d / kBK;
  const int r = (kRole == kRoleLse || a.scratch) ? int(blockIdx.y) : a.r;
  const int64_t Mside = kRole == kRoleDy ? a.C : a.N;
  const int64_t Kside = kRole == kRoleDy ? a.N : a.C;
  const int64_t m0 = int64_t(blockIdx.x) * kBM;
  int64_t k0a;
  int nK;
  k_range<kRole>(a, m0, k0a, nK);
  const uint32_t vb = uint32_t(v_bytes(d));

  if (threadIdx.x == 0) {
    for (int i = 0; i < kAB; ++i) {
      mbar_init(&ctl.ab_full[i], 1);
      mbar_init(&ctl.ab_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.s_full[i], 1);
      mbar_init(&ctl.s_empty[i], kEpiWarps);
      mbar_init(&ctl.v_full[i], 1);
      mbar_init(&ctl.v_empty[i], 1);
    }
    mbar_init(&ctl.p_full, kEpiWarps);
    mbar_init(&ctl.p_empty, 1);
    mbar_init(&ctl.done, 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  const uint32_t tcols = kGrad ? 512u : 256u;
  if (warp == 1) {
    tmem_alloc(&ctl.tmem_base, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  volatile int* abortp = &ctl.abort;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      if (kGrad) prefetch_tmap(&tmV);
      const int32_t arow = int32_t(int64_t(r) * Mside + m0);
      uint32_t it = 0;
      int nv_issued = 0;
      bool ok = true;
      for (int kt = 0; kt < nK && ok && !*abortp; ++kt) {
        const int32_t brow = int32_t(int64_t(r) * Kside + k0a + int64_t(kt) * kBN);
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int st = int(it % kAB);
          if (!mbar_wait(&ctl.ab_empty[st], ((it / kAB) & 1u) ^ 1u, &ctl.abort, kTimeoutNs)) {
            on_timeout(ctl, a.status);
            ok = false;
            break;
          }
          uint8_t* sa = ab + size_t(st) * 2 * kSlab;
          mbar_arrive_expect_tx(&ctl.ab_full[st], 2 * kSlab);
          tma_load_2d(sa, &tmA, &ctl.ab_full[st], ks * kBK, arow);
          tma_load_2d(sa + kSlab, &tmB, &ctl.ab_full[st], ks * kBK, brow);
        }
        if (kGrad && ok) {
          const int vs = kt % a.nv;
          if (!mbar_wait(&ctl.v_empty[vs], ((kt / a.nv) & 1) ^ 1, &ctl.abort, kTimeoutNs)) {
            on_timeout(ctl, a.status);
            ok = false;
            break;
          }
          uint8_t* sv = vbuf + size_t(vs) * vb;
          const int32_t kx = int32_t(k0a + int64_t(kt) * kBN);
          mbar_arrive_expect_tx(&ctl.v_full[vs], vb);
          // two K atoms of 64 positions, each d/64 boxes of 64 columns (8 KB apart)
          for (int at = 0; at < 2; ++at)
            for (int h = 0; h < d; h += 64)
              tma_load_3d(sv + at * (vb / 2) + size_t(h) * 128, &tmV, &ctl.v_full[vs], h,
                          kx + at * kBK, r);
          ++nv_issued;
        }
      }
      // every issued copy has landed before the CTA may exit
      for (uint32_t j = (it > kAB ? it - kAB : 0); j < it; ++j)
        mbar_wait_limit(&ctl.ab_full[j % kAB], (j / kAB) & 1u, kTimeoutNs);
      if (kGrad)
        for (int j = (nv_issued > a.nv ? nv_issued - a.nv : 0); j < nv_issued; ++j)
          mbar_wait_limit(&ctl.v_full[j % a.nv], (j / a.nv) & 1, kTimeoutNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kBM, kBN);
      const uint32_t idesc_o = idesc_bf16_f32_bmn(kBM, d);  // V MN-major
      uint32_t it = 0;
      bool ok = true;
      auto mma_pv = [&](int j) {  // O += P_j V_j (hi and lo halves)
        if (!mbar_wait(&ctl.p_full, uint32_t(j) & 1u, &ctl.abort, kTimeoutNs) ||
            !mbar_wait(&ctl.v_full[j % a.nv], (j / a.nv) & 1, &ctl.abort, kTimeoutNs)) {
          on_timeout(ctl, a.status);
          ok = false;
          return;
        }
        tc_fence_after();
        const uint8_t* sv = vbuf + size_t(j % a.nv) * vb;
#pragma unroll
        for (int at = 0; at < 2; ++at) {
          const uint64_t dh = desc_k_sw128(smem_u32(phi + at * kSlab));
          const uint64_t dl = desc_k_sw128(smem_u32(plo + at * kSlab));
          const uint64_t dv = desc_mn_sw128(smem_u32(sv + at * (vb / 2)), 8192u);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {  // 16 K rows of 128 B per MMA
            mma_bf16(tmem + 256, dh + 2 * kk, dv + 128u * kk, idesc_o, (j | at | kk) != 0);
            mma_bf16(tmem + 256, dl + 2 * kk, dv + 128u * kk, idesc_o, 1);
          }
        }
        mma_commit(&ctl.p_empty);
        mma_commit(&ctl.v_empty[j % a.nv]);
      };
      for (int kt = 0; kt < nK && ok && !*abortp; ++kt) {
        const int sb = kt & 1;
        if (!mbar_wait(&ctl.s_empty[sb], ((kt >> 1) & 1) ^ 1, &ctl.abort, kTimeoutNs)) {
          on_timeout(ctl, a.status);
          ok = false;
          break;
        }
        tc_fence_after();
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int st = int(it % kAB);
          if (!mbar_wait(&ctl.ab_full[st], (it / kAB) & 1u, &ctl.abort, kTimeoutNs)) {
            on_timeout(ctl, a.status);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* sa = ab + size_t(st) * 2 * kSlab;
          const uint64_t da = desc_k_sw128(smem_u32(sa));
          const uint64_t db = desc_k_sw128(smem_u32(sa + kSlab));
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16(tmem + uint32_t(sb * kBN), da + 2 * kk, db + 2 * kk, idesc_s,
                     (ks | kk) != 0);
          mma_commit(&ctl.ab_empty[st]);
        }
        if (!ok) break;
        mma_commit(&ctl.s_full[sb]);
        if (kGrad && kt >= 1) mma_pv(kt - 1);
      }
      if (kGrad && ok && nK >= 1 && !*abortp) mma_pv(nK - 1);
      mma_commit(&ctl.done);
      mbar_wait_limit(&ctl.done, 0, kTimeoutNs);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int g = (warp - 2) >> 2;  // warpgroup: columns 32g..32g+31 of every score tile
    const int q4 = warp & 3;        // TMEM lane quarter this warp may read
    const int m = q4 * 32 + lane;   // this thread's position in the M tile
    const int64_t mi = m0 + m;
    const bool mvalid = mi < Mside;
    const int n_r = kR ? kR : a.n_r, n_ec = a.n_ec;
    const int o = kR == 2 ? 1 - r : 0;  // the other round (two rounds)
    const int64_t rN = int64_t(r) * a.N;
    // This thread's own side.  Rows (LSE, DX): window, positive, lse, and the row's chunk
    // in every round; items (DY): the item's chunk in every round.
    int64_t w0 = 0, w1 = 0;
    int64_t my_pz = -1;
    float my_nl = 0.0f;  // -lse * log2(e)
    int32_t myc_r = 0, myc_o = 0;
    int32_t myc[kR == 0 ? kMaxRounds : 1];
    const int32_t* own = kRole == kRoleDy ? a.itemc : a.rowc;
    const int64_t ownM = kRole == kRoleDy ? a.C : a.N;
    if (mvalid) {
      if (kRole != kRoleDy) {
        const int64_t cm = chunk_of(mi, a.N, a.n_c);
        w0 = chunk_start(cm - n_ec < 0 ? 0 : cm - n_ec, a.C, a.n_c);
        w1 = chunk_start(cm + n_ec + 1 > a.n_c ? a.n_c : cm + n_ec + 1, a.C, a.n_c);
        my_pz = a.pz[rN + mi];
        if (kRole == kRoleDx) my_nl = -a.lse_sorted[rN + mi] * kLog2e;
      } else {
        myc_r = int32_t(chunk_of(mi, a.C, a.n_c));
      }
      if (kR == 2) myc_o = own[(int64_t(r) * 2 + o) * ownM + mi];
    }
    if (kR == 0) {
#pragma unroll
      for (int s2 = 0; s2 < (kR == 0 ? kMaxRounds : 1); ++s2)
        myc[s2] = (s2 < n_r && mvalid) ? own[(int64_t(r) * n_r + s2) * ownM + mi] : 0;
    }
    const int32_t* oc_tab = kRole == kRoleDy ? a.rowc : a.itemc;  // the other side's chunks
    // Column metadata of every K tile, staged in shared memory (two buffers) by all
    // epilogue threads, each tile's loads issued one tile ahead:
    //   kR = 1, 2: DY one int4 per column (row's chunk in round r, its positive's
    //              position, its lse, its chunk in the other round); LSE / DX one int per
    //              column (the item's chunk in the other round; none for one round);
    //   kR = 0:    [round][column] chunks (and, DY, [n_r] positives, [n_r + 1] lse).
    const int n_meta = kR == 0 ? (kRole == kRoleDy ? (n_r + 2) * kBN : n_r * kBN)
                               : (kRole == kRoleDy ? 4 * kBN : (kR == 2 ? kBN : 0));
    const int et = threadIdx.x - 64;
    int32_t pre[kMetaPer];
    auto meta_load = [&](int t) {
#pragma unroll
      for (int j = 0; j < kMetaPer; ++j) {
        const int v = et + j * kEpiThreads;
        pre[j] = 0;
        if (v >= n_meta || t >= nK) continue;
        int arr, c;
        if (kR != 0 && kRole == kRoleDy) {  // packed: field v & 3 of column v >> 2
          arr = v & 3;
          c = v >> 2;
        } else {
          arr = v >> 7;
          c = v & (kBN - 1);
        }
        const int64_t kk = k0a + int64_t(t) * kBN + c;
        if (kk >= Kside) continue;
        if (kR != 0) {
          if (kRole == kRoleDy) {
            if (arr == 0) pre[j] = __ldg(a.rowc + (int64_t(r) * n_r + r) * a.N + kk);
            else if (arr == 1) pre[j] = __ldg(a.pz + rN + kk);
            else if (arr == 2) pre[j] = __float_as_int(-__ldg(a.lse_sorted + rN + kk) * kLog2e);
            else if (kR == 2) pre[j] = __ldg(a.rowc + (int64_t(r) * 2 + o) * a.N + kk);
          } else {
            pre[j] = __ldg(a.itemc + (int64_t(r) * 2 + o) * a.C + kk);
          }
        } else if (arr < n_r) {
          if (kRole != kRoleDy && arr == r) continue;  // a row's own round: positions decide
          pre[j] = __ldg(oc_tab + (int64_t(r) * n_r + arr) * Kside + kk);
        } else if (arr == n_r) {
          pre[j] = __ldg(a.pz + rN + kk);
        } else {
          pre[j] = __float_as_int(-__ldg(a.lse_sorted + rN + kk) * kLog2e);
        }
      }
    };
    auto meta_store = [&](int t) {
      int32_t* dst = ctl.meta[t & 1];
#pragma unroll
      for (int j = 0; j < kMetaPer; ++j)
        if (et + j * kEpiThreads < n_meta) dst[et + j * kEpiThreads] = pre[j];
    };
    meta_load(0);
    meta_store(0);
    meta_load(1);
    named_barrier(1, kEpiThreads);
    float run_m = -INFINITY, run_s = 0.0f;  // LSE: online max (log2 units) and sum
    const uint32_t trow = tmem + (uint32_t(q4 * 32) << 16);
    const int col0 = 32 * g;
    bool ok = true;
    // Every epilogue thread runs every iteration to the named barrier at its end, also
    // after a timed-out wait (then without touching TMEM or the tiles).
    for (int kt = 0; kt < nK; ++kt) {
      const int sb = kt & 1;
      bool got = ok && mbar_wait(&ctl.s_full[sb], (kt >> 1) & 1, &ctl.abort, kTimeoutNs);
      got = __all_sync(0xFFFFFFFFu, got);  // the warp's TMEM load is collective
      if (!got && ok) {
        if (lane == 0) on_timeout(ctl, a.status);
        ok = false;
      }
      if (ok) {
        tc_fence_after();
        float v[32];
        tmem_load32(trow + uint32_t(sb * kBN + col0), v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.s_empty[sb]);
        const int32_t* md = ctl.meta[kt & 1];
        const int64_t kb = k0a + int64_t(kt) * kBN + col0;  // K index of v[0]
        // the live columns of this block: [lo, hi) minus the positive's column
        int lo = 0, hi = 0, pzc = -1;
        if (mvalid) {
          if (kRole == kRoleDy) {
            const int64_t rest = a.N - kb;
            hi = rest <= 0 ? 0 : (rest >= 32 ? 32 : int(rest));
          } else {
            const int64_t l = w0 - kb, h = w1 - kb;
            lo = l <= 0 ? 0 : (l >= 32 ? 32 : int(l));
            hi = h <= 0 ? 0 : (h >= 32 ? 32 : int(h));
            if (my_pz >= kb && my_pz < kb + 32) pzc = int(my_pz - kb);
          }
        }
        // v[u] becomes, per live column, log2(e) times the score plus (gradient roles)
        // the row's -lse * log2(e); w[u] the column's weight 1/cnt (0: dead)
        float w[kGrad ? 1 : 32];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const int c = col0 + u;
          bool live = u >= lo && u < hi && u != pzc;
          float nl = my_nl;
          float wt = 1.0f;
          if (kRole == kRoleDy && kR != 0) {
            const int4 mc = reinterpret_cast<const int4*>(md)[c];
            live = live && abs(mc.x - myc_r) <= n_ec && mc.y != int32_t(mi);
            nl = __int_as_float(mc.z);
            if (kR == 2 && abs(mc.w - myc_o) <= n_ec) wt = 0.5f;
          } else if (kRole == kRoleDy) {
            live = live && abs(md[r * kBN + c] - myc_r) <= n_ec && md[n_r * kBN + c] != int32_t(mi);
            nl = __int_as_float(md[(n_r + 1) * kBN + c]);
          } else if (kR == 2) {
            if (abs(md[c] - myc_o) <= n_ec) wt = 0.5f;
          }
          if (kR == 0) {
            int cnt = 1;
            for (int s2 = 0; s2 < n_r; ++s2)
              if (s2 != r && abs(md[s2 * kBN + c] - myc[s2]) <= n_ec) ++cnt;
            wt = __fdividef(1.0f, float(cnt));
          }
          if (kGrad) {
            v[u] = live ? wt * ex2(fmaf(v[u], kLog2e, nl)) : 0.0f;  // p / cnt
          } else {
            w[u] = live ? wt : 0.0f;
            v[u] = live ? fmaf(v[u], kLog2e, nl) : -INFINITY;
          }
        }
        if (kRole == kRoleLse) {
          float bm = -INFINITY;
#pragma unroll
          for (int u = 0; u < 32; ++u) bm = fmaxf(bm, v[u]);
          if (bm != -INFINITY) {
            if (bm > run_m) {
              run_s *= ex2(run_m - bm);
              run_m = bm;
            }
            float acc = 0.0f;
#pragma unroll
            for (int u = 0; u < 32; ++u) acc = fmaf(w[u], ex2(v[u] - run_m), acc);
            run_s += acc;
          }
        } else {
          // P into the shared tiles once the previous product has read them
          got = mbar_wait(&ctl.p_empty, uint32_t(kt & 1) ^ 1u, &ctl.abort, kTimeoutNs);
          if (!__all_sync(0xFFFFFFFFu, got)) {
            if (lane == 0) on_timeout(ctl, a.status);
            ok = false;
          } else {
            uint8_t* th = phi + (col0 >> 6) * kSlab;
            uint8_t* tl = plo + (col0 >> 6) * kSlab;
            const int cb = (col0 & 63) >> 3;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t h[4], l[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float x0 = v[8 * j + 2 * e], x1 = v[8 * j + 2 * e + 1];
                const __nv_bfloat162 hb = __floats2bfloat162_rn(x0, x1);
                const float2 hf = __bfloat1622float2(hb);
                const __nv_bfloat162 lb = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
                h[e] = *reinterpret_cast<const uint32_t*>(&hb);
                l[e] = *reinterpret_cast<const uint32_t*>(&lb);
              }
              *reinterpret_cast<uint4*>(th + sw128_chunk(m, cb + j)) =
                  make_uint4(h[0], h[1], h[2], h[3]);
              *reinterpret_cast<uint4*>(tl + sw128_chunk(m, cb + j)) =
                  make_uint4(l[0], l[1], l[2], l[3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.p_full);
          }
        }
      }
      // tile kt+1's metadata in (its buffer was last read during tile kt-1, which every
      // thread finished before the barrier that ended it); tile kt+2's loads out
      meta_store(kt + 1);
      meta_load(kt + 2);
      named_barrier(1, kEpiThreads);
    }
    if (kRole == kRoleLse) {
      // the four warpgroups' partials of every row
      ctl.part_m[g][m] = run_m;
      ctl.part_s[g][m] = run_s;
      named_barrier(1, kEpiThreads);
      if (g == 0 && mvalid) {
        float M = -INFINITY, S = 0.0f;  // M in log2 units, as the partials
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (ctl.part_s[w][m] > 0.0f) M = fmaxf(M, ctl.part_m[w][m]);
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (ctl.part_s[w][m] > 0.0f) S += ctl.part_s[w][m] * ex2(ctl.part_m[w][m] - M);
        a.ms[rN + mi] = make_float2(S > 0.0f ? M / kLog2e : 0.0f, S);
      }
    } else {
      bool fin = ok && mbar_wait(&ctl.done, 0, &ctl.abort, kTimeoutNs) && nK > 0;
      fin = __all_sync(0xFFFFFFFFu, fin);
      tc_fence_after();
      if (fin) {
        const float scale = a.dloss[0] / float(a.N);
        const int64_t dst = mvalid ? a.perm[int64_t(r) * Mside + mi] : 0;
        float* o = a.out + dst * d;
        for (int oc = col0; oc < d; oc += 128) {
          float v[32];
          tmem_load32(trow + 256u + uint32_t(oc), v);
          if (mvalid && a.scratch) {  // this round's part, written; the rounds add later
            float4* q = reinterpret_cast<float4*>(a.scratch + (rN + dst) * d + oc);
#pragma unroll
            for (int u = 0; u < 8; ++u)
              q[u] = make_float4(scale * v[4 * u], scale * v[4 * u + 1], scale * v[4 * u + 2],
                                 scale * v[4 * u + 3]);
          } else if (mvalid) {
            float4* q = reinterpret_cast<float4*>(o + oc);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              float4 x = q[u];
              x.x = fmaf(scale, v[4 * u], x.x);
              x.y = fmaf(scale, v[4 * u + 1], x.y);
              x.z = fmaf(scale, v[4 * u + 2], x.z);
              x.w = fmaf(scale, v[4 * u + 3], x.w);
              q[u] = x;
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}


template <int kRole, int kR>
cudaError_t run_window_r(const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& V,
                         const Args& a, unsigned gx, unsigned gy, cudaStream_t st) {
  size_t smem = window_smem(kRole, a.d, a.nv);
  // at most two CTAs per SM: their TMEM allocations (256 columns each in the LSE role,
  // 512 in the gradient roles, one CTA) always fit
  if (smem < 80 * 1024) smem = 80 * 1024;
  cudaError_t e = cudaFuncSetAttribute(k_window_tc<kRole, kR>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  k_window_tc<kRole, kR><<<dim3(gx, gy), kThreads, smem, st>>>(A, B, V, a);
  count_launches(1);
  return cudaGetLastError();
}

template <int kRole>
cudaError_t run_window(const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& V,
                       const Args& a, unsigned gx, unsigned gy, cudaStream_t st) {
  if (a.n_r == 1) return run_window_r<kRole, 1>(A, B, V, a, gx, gy, st);
  if (a.n_r == 2) return run_window_r<kRole, 2>(A, B, V, a, gx, gy, st);
  return run_window_r<kRole, 0>(A, B, V, a, gx, gy, st);
}

Args base_args(const rece_plan_s& p, const int32_t* itemc, const int32_t* rowc,
               const int32_t* pz, uint32_t* status) {
  const auto& c = p.cfg;
  Args a{};
  a.N = c.N;
  a.C = c.C;
  a.d = c.d;
  a.n_c = c.n_c;
  a.n_ec = c.n_ec;
  a.n_r = c.n_r;
  a.nv = c.d <= 128 ? 2 : 1;
  a.itemc = itemc;
  a.rowc = rowc;
  a.pz = pz;
  a.status = status;
  return a;
}

}  // namespace

bool window_tc_supported(const rece_plan_s& p) {
  return p.use_tc && p.cfg.d <= 256 && p.cfg.n_r <= kMaxRounds;
}

cudaError_t launch_window_lse_tc(const rece_plan_s& p, const void* Xs, const void* Ys,
                                 const int32_t* itemc, const int32_t* rowc, const int32_t* pz,
                                 float2* ms, uint32_t* status, cudaStream_t st) {
  const auto& c = p.cfg;
  if (c.N == 0) return cudaSuccess;
  CUtensorMap tA, tB;
  cudaError_t e = make_tmap_bf16(&tA, Xs, uint64_t(c.n_r) * c.N, c.d, kBM);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tB, Ys, uint64_t(c.n_r) * c.C, c.d, kBN);
  if (e != cudaSuccess) return e;
  Args a = base_args(p, itemc, rowc, pz, status);
  a.ms = ms;
  return run_window<kRoleLse>(tA, tB, tB, a, unsigned(ceil_div(c.N, kBM)), unsigned(c.n_r), st);
}

cudaError_t launch_window_grad_tc(const rece_plan_s& p, bool dy, const void* Xs,
                                  const void* Ys, const int32_t* itemc, const int32_t* rowc, const int32_t* pz,
                                  const float* lse_sorted, const int32_t* perm,
                                  const float* dloss, float* out, float* scratch,
                                  uint32_t* status, cudaStream_t st) {
  const auto& c = p.cfg;
  if (c.N == 0) return cudaSuccess;
  CUtensorMap tX, tY, tV;
  cudaError_t e = make_tmap_bf16(&tX, Xs, uint64_t(c.n_r) * c.N, c.d, kBM);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tY, Ys, uint64_t(c.n_r) * c.C, c.d, kBM);
  if (e != cudaSuccess) return e;
  // V: the sorted rows of X (dY) or Y (dX) of every round, read MN-major
  if (dy)
    e = make_tmap_bf16_3d(&tV, Xs, uint64_t(c.d), uint64_t(c.N), uint64_t(c.n_r), kBK);
  else
    e = make_tmap_bf16_3d(&tV, Ys, uint64_t(c.d), uint64_t(c.C), uint64_t(c.n_r), kBK);
  if (e != cudaSuccess) return e;
  Args a = base_args(p, itemc, rowc, pz, status);
  a.lse_sorted = lse_sorted;
  a.perm = perm;
  a.dloss = dloss;
  a.out = out;
  if (!dy && scratch) {
    // dX: every round in one grid (the rows' tiles alone would not fill the GPU), each
    // writing its part; then the parts are added into dX in round order
    a.scratch = scratch;
    e = run_window<kRoleDx>(tX, tY, tV, a, unsigned(ceil_div(c.N, kBM)), unsigned(c.n_r), st);
    if (e != cudaSuccess) return e;
    return launch_add_parts(scratch, c.N * int64_t(c.d), c.n_r, out, st);
  }
  for (int r = 0; r < c.n_r; ++r) {  // rounds in order: each adds into the same rows
    a.r = r;
    e = dy ? run_window<kRoleDy>(tY, tX, tV, a, unsigned(ceil_div(c.C, kBM)), 1u, st)
           : run_window<kRoleDx>(tX, tY, tV, a, unsigned(ceil_div(c.N, kBM)), 1u, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace rece
