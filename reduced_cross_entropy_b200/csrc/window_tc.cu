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
//        O += P V with V = the K tile of the d-major sorted catalogue copy; at the end
//        dX[row] += O * dloss / N.
//   DY   M = items, K = rows.  The same with the roles swapped (the pair is live when the
//        item lies in the row's window), V = the d-major sorted copy of X; dY[item] +=.
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

struct Ctl {
  uint64_t ab_full[kAB], ab_empty[kAB];
  uint64_t s_full[2], s_empty[2];
  uint64_t v_full[2], v_empty[2];
  uint64_t p_full, p_empty;
  uint64_t done;
  uint32_t tmem_base;
  int abort;
  float part_m[4][kBM], part_s[4][kBM];  // LSE: the warpgroups' partial (max, sum)
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

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  return uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(a))) |
         (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(b))) << 16);
}

// The K range of an M tile: the union of the windows of its 128 positions, as a start
// rounded down to 64 (TMA column coordinates of the d-major copies stay 16-byte aligned)
// and a count of 128-wide tiles.
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

template <int kRole>
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
  const int r = kRole == kRoleLse ? int(blockIdx.y) : a.r;
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
          tma_load_2d(sv, &tmV, &ctl.v_full[vs], kx, r * d);
          tma_load_2d(sv + vb / 2, &tmV, &ctl.v_full[vs], kx + kBK, r * d);
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
      const uint32_t idesc_o = idesc_bf16_f32(kBM, d);
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
          const uint64_t dv = desc_k_sw128(smem_u32(sv + at * (vb / 2)));
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            mma_bf16(tmem + 256, dh + 2 * kk, dv + 2 * kk, idesc_o, (j | at | kk) != 0);
            mma_bf16(tmem + 256, dl + 2 * kk, dv + 2 * kk, idesc_o, 1);
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
    const int n_r = a.n_r, n_ec = a.n_ec;
    const int64_t rN = int64_t(r) * a.N;
    // this thread's own side: window, positive and lse of a row (LSE, DX); its chunk in
    // every round (rows: rowc, items: itemc)
    int64_t w0 = 0, w1 = 0;
    int32_t my_pz = -1;
    float my_lse = 0.0f;
    int32_t myc[kMaxRounds];
    if (mvalid && kRole != kRoleDy) {
      const int64_t cm = chunk_of(mi, a.N, a.n_c);
      w0 = chunk_start(cm - n_ec < 0 ? 0 : cm - n_ec, a.C, a.n_c);
      w1 = chunk_start(cm + n_ec + 1 > a.n_c ? a.n_c : cm + n_ec + 1, a.C, a.n_c);
      my_pz = a.pz[rN + mi];
      if (kRole == kRoleDx) my_lse = a.lse_sorted[rN + mi];
    }
#pragma unroll
    for (int s2 = 0; s2 < kMaxRounds; ++s2) {
      myc[s2] = 0;
      if (s2 < n_r && mvalid)
        myc[s2] = kRole == kRoleDy ? a.itemc[(int64_t(r) * n_r + s2) * a.C + mi]
                                   : a.rowc[(int64_t(r) * n_r + s2) * a.N + mi];
    }
    const int32_t* oc_tab = kRole == kRoleDy ? a.rowc : a.itemc;  // the other side's chunks
    const int64_t oc_M = kRole == kRoleDy ? a.N : a.C;
    float run_m = -INFINITY, run_s = 0.0f;  // LSE: online max and sum
    const uint32_t trow = tmem + (uint32_t(q4 * 32) << 16);
    const int col0 = 32 * g;
    bool ok = true;
    for (int kt = 0; kt < nK; ++kt) {
      const int sb = kt & 1;
      bool got = ok && mbar_wait(&ctl.s_full[sb], (kt >> 1) & 1, &ctl.abort, kTimeoutNs);
      got = __all_sync(0xFFFFFFFFu, got);  // the warp's TMEM load is collective
      if (!got) {
        if (ok && lane == 0) on_timeout(ctl, a.status);
        ok = false;
        break;
      }
      tc_fence_after();
      float v[32];
      tmem_load32(trow + uint32_t(sb * kBN + col0), v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.s_empty[sb]);
      const int64_t kb = k0a + int64_t(kt) * kBN + col0;  // K index of v[0]
      // v[u] becomes the column's weight 1/cnt times exp(s - lse) (gradient roles), or
      // its weight alone with -1 for a dead column (LSE)
      float wgt[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int64_t kk = kb + u;
        bool live;
        float lse_k = my_lse;
        if (kRole == kRoleDy) {  // kk is a sorted row, this thread an item
          live = mvalid && kk < a.N;
          if (live)
            live = abs(__ldg(a.rowc + (int64_t(r) * n_r + r) * a.N + kk) - myc[r]) <= n_ec &&
                   __ldg(a.pz + rN + kk) != int32_t(mi);
          if (live) lse_k = __ldg(a.lse_sorted + rN + kk);
        } else {  // kk is a sorted catalogue position, this thread a row
          live = mvalid && kk >= w0 && kk < w1 && kk != my_pz;
        }
        float cnt = 1.0f;
        if (live && n_r > 1) {
          for (int s2 = 0; s2 < n_r; ++s2)
            if (s2 != r &&
                abs(__ldg(oc_tab + (int64_t(r) * n_r + s2) * oc_M + kk) - myc[s2]) <= n_ec)
              cnt += 1.0f;
        }
        wgt[u] = live ? 1.0f / cnt : 0.0f;
        if (kGrad) v[u] = live ? expf(v[u] - lse_k) * wgt[u] : 0.0f;
      }
      if (kRole == kRoleLse) {
        float bm = -INFINITY;
#pragma unroll
        for (int u = 0; u < 32; ++u)
          if (wgt[u] > 0.0f) bm = fmaxf(bm, v[u]);
        if (bm > run_m) {
          run_s *= expf(run_m - bm);
          run_m = bm;
        }
#pragma unroll
        for (int u = 0; u < 32; ++u)
          if (wgt[u] > 0.0f) run_s += expf(v[u] - run_m) * wgt[u];
        continue;
      }
      // gradient roles: P into the shared tiles once the previous product has read them
      got = mbar_wait(&ctl.p_empty, uint32_t(kt & 1) ^ 1u, &ctl.abort, kTimeoutNs);
      if (!__all_sync(0xFFFFFFFFu, got)) {
        if (lane == 0) on_timeout(ctl, a.status);
        ok = false;
        break;
      }
      uint8_t* th = phi + (col0 >> 6) * kSlab;
      uint8_t* tl = plo + (col0 >> 6) * kSlab;
      const int cb = (col0 & 63) >> 3;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = v[8 * j + 2 * e], x1 = v[8 * j + 2 * e + 1];
          const float h0 = __bfloat162float(__float2bfloat16_rn(x0));
          const float h1 = __bfloat162float(__float2bfloat16_rn(x1));
          h[e] = pack_bf16(h0, h1);
          l[e] = pack_bf16(x0 - h0, x1 - h1);
        }
        *reinterpret_cast<uint4*>(th + sw128_chunk(m, cb + j)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(tl + sw128_chunk(m, cb + j)) = make_uint4(l[0], l[1], l[2], l[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.p_full);
    }
    if (kRole == kRoleLse) {
      // the four warpgroups' partials of every row
      ctl.part_m[g][m] = run_m;
      ctl.part_s[g][m] = run_s;
      named_barrier(1, kEpiThreads);
      if (g == 0 && mvalid) {
        float M = -INFINITY, S = 0.0f;
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (ctl.part_s[w][m] > 0.0f) M = fmaxf(M, ctl.part_m[w][m]);
#pragma unroll
        for (int w = 0; w < 4; ++w)
          if (ctl.part_s[w][m] > 0.0f) S += ctl.part_s[w][m] * expf(ctl.part_m[w][m] - M);
        a.ms[rN + mi] = make_float2(S > 0.0f ? M : 0.0f, S);
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
          if (mvalid) {
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


template <int kRole>
cudaError_t run_window(const CUtensorMap& A, const CUtensorMap& B, const CUtensorMap& V,
                       const Args& a, unsigned gx, unsigned gy, cudaStream_t st) {
  size_t smem = window_smem(kRole, a.d, a.nv);
  // at most two CTAs per SM: their TMEM allocations (256 columns each in the LSE role,
  // 512 in the gradient roles, one CTA) always fit
  if (smem < 80 * 1024) smem = 80 * 1024;
  cudaError_t e = cudaFuncSetAttribute(k_window_tc<kRole>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  k_window_tc<kRole><<<dim3(gx, gy), kThreads, smem, st>>>(A, B, V, a);
  count_launches(1);
  return cudaGetLastError();
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
                                  const void* Ys, const void* XsT, const void* YsT,
                                  const int32_t* itemc, const int32_t* rowc, const int32_t* pz,
                                  const float* lse_sorted, const int32_t* perm,
                                  const float* dloss, float* out, uint32_t* status,
                                  cudaStream_t st) {
  const auto& c = p.cfg;
  if (c.N == 0) return cudaSuccess;
  CUtensorMap tX, tY, tV;
  cudaError_t e = make_tmap_bf16(&tX, Xs, uint64_t(c.n_r) * c.N, c.d, kBM);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&tY, Ys, uint64_t(c.n_r) * c.C, c.d, kBM);
  if (e != cudaSuccess) return e;
  if (dy)
    e = make_tmap_bf16_ld(&tV, XsT, uint64_t(c.n_r) * c.d, c.N, p.ld_n, uint32_t(c.d));
  else
    e = make_tmap_bf16_ld(&tV, YsT, uint64_t(c.n_r) * c.d, c.C, p.ld_c, uint32_t(c.d));
  if (e != cudaSuccess) return e;
  Args a = base_args(p, itemc, rowc, pz, status);
  a.lse_sorted = lse_sorted;
  a.perm = perm;
  a.dloss = dloss;
  a.out = out;
  for (int r = 0; r < c.n_r; ++r) {  // rounds in order: each adds into the same rows
    a.r = r;
    e = dy ? run_window<kRoleDy>(tY, tX, tV, a, unsigned(ceil_div(c.C, kBM)), 1u, st)
           : run_window<kRoleDx>(tX, tY, tV, a, unsigned(ceil_div(c.N, kBM)), 1u, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace rece
