// bwd_tc.cu -- dX of step 6 on the tcgen05 tensor cores (bf16 mode): the row gradients of
// the reduced loss (RECE, equation 4, over the positive and the kept negatives, selection
// held constant) as dense block products of the sparse coefficient matrix.
//
//   g_ij = (exp(l_ij - lse_i) - [j == z_i]) * dloss / N,   dX_i = sum_j g_ij y_j
//
// The negatives of round r of a row all lie in that row's window of round r's sorted
// catalogue, so per round the coefficients form a band: rows of chunk c against the
// sorted positions of chunks c-n_ec..c+n_ec.  With G_r that band (sorted rows x sorted
// positions, the round's kept entries only -- the merge kept each pair once, in the
// earliest round whose window holds it):
//
//   dX[rows] += G_r[rows, window] Ys_r[window]     (work item: 128 sorted rows)
//
// A work item streams its window in slabs of 64 positions: four builder warps write the
// slab's 128 x 64 tile of G into shared memory in the 128-byte-swizzled K-major layout
// (zeros, then the row's entries of the slab, which come grouped by slab) while TMA brings
// the matching 64 rows of the sorted copy Ys (64-column boxes, which the MMA reads as an
// MN-major B operand: no transposed copy) and one thread issues
// tcgen05.mma into TMEM accumulators of 128 x NS fp32 (NS <= 512 columns of d per CTA:
// two accumulators of N = 256 past 256).
// The tiles hold the negatives' softmax probabilities p_ij = exp(l_ij - lse_i), which the
// merge stored split as hi + lo, both bf16 (hi = bf16(p), lo = bf16(p - hi)); both halves
// are multiplied, so about 16 bits of p survive against 8 for a plain bf16 tile, and the
// epilogue applies the factor dloss / N.
//
// This pays where gathering the catalogue rows does not: at large d, or when the sorted
// catalogue does not fit in L2.  The transposed product for dY, G_r^T Xs_r per tile of
// positions (k_bwd_dy_tc below), pays only at large d (d >= 1024): its K ranges are short
// and every slice of d rebuilds the same tiles, against a pair sort and gather whose cost
// per pair grows with d.
//
// Determinism: each dX row is written by one CTA per launch, in a fixed K order; the
// positive term is written first (dX_i = g_iz y_z), then the rounds add in round order.
#include <cmath>

#include "common.cuh"
#include "plan.h"
#include "sm100.cuh"
#include "tc.h"

#define RECE_TRY(x)                          \
  do {                                       \
    const cudaError_t err_ = (x);            \
    if (err_ != cudaSuccess) return err_;    \
  } while (0)

namespace rece {
namespace {

using namespace sm100;

constexpr int kBM = 128;           // rows of G (dX) or of G^T (dY) per work item
constexpr int kBK = 64;            // K per slab
constexpr int kAStages = 2;        // G tiles being built / consumed
constexpr int kMaxBStages = 8;     // TMA slabs in flight
constexpr int kBuilders = 128;     // warps 0-3: builders, then the epilogue
constexpr int kThreads = kBuilders + 64;  // warp 4: TMA producer, warp 5: MMA issuer
constexpr uint32_t kATile = kBM * kBK * 2;  // one bf16 G tile (16 KB)
constexpr uint64_t kTimeoutNs = 1000000000ull;

struct Ctl {
  uint64_t bfull[kMaxBStages], bempty[kMaxBStages];
  uint64_t afull[kAStages], aempty[kAStages];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

// Dynamic shared memory: A_hi[kAStages], A_lo[kAStages], B[nb] (NS x 128 B each), Ctl.
__host__ __device__ constexpr size_t smem_bytes(int nb, int ns) {
  return 1024 + size_t(2 * kAStages) * kATile + size_t(nb) * ns * 128 + sizeof(Ctl);
}

// Byte offset of element (row, col) of a 128 x 64 bf16 tile in the 128-byte-swizzled
// K-major layout (what a TMA box {64, rows} with SWIZZLE_128B writes): rows of 128 B in
// 8-row atoms of 1024 B, the 16-byte chunk index xor-ed with row % 8.
__device__ __forceinline__ uint32_t sw128_offset(int row, int col) {
  return uint32_t((row >> 3) * 1024 + (row & 7) * 128 + ((((col >> 3) ^ row) & 7) << 4) +
                  (col & 7) * 2);
}

// Zeros one 128-byte row; the chunk order is rotated by the row so that the lanes of a
// warp (32 consecutive rows, 128 B apart) spread over all banks.
__device__ __forceinline__ void zero_row(uint8_t* tile, int row) {
  uint4* p = reinterpret_cast<uint4*>(tile + (row >> 3) * 1024 + (row & 7) * 128);
#pragma unroll
  for (int j = 0; j < 8; ++j) p[(j + row) & 7] = make_uint4(0u, 0u, 0u, 0u);
}


// The dX kernel's G tiles use the K-major layout without swizzle instead: 8 x 16-byte
// core matrices, the 8 of a row group along K 128 B apart (leading byte offset), row
// groups 1024 B apart (stride byte offset).  Element (row, col) then sits in bank
// 4 (row % 8) + (col % 8) / 2, so the lanes of a warp (32 consecutive rows, one entry
// each) can only collide four at a time, where the 128-byte swizzle spreads their random
// columns over all 32 banks.
__device__ __forceinline__ uint32_t plain_offset(int row, int col) {
  return uint32_t((row >> 3) * 1024 + (col >> 3) * 128 + (row & 7) * 16 + (col & 7) * 2);
}
__device__ __forceinline__ void zero_row_plain(uint8_t* tile, int row) {
  uint8_t* p = tile + (row >> 3) * 1024 + (row & 7) * 16;
#pragma unroll
  for (int j = 0; j < 8; ++j) *reinterpret_cast<uint4*>(p + j * 128) = make_uint4(0u, 0u, 0u, 0u);
}
// A 16-bit shared store that only happens when `p` holds (one predicated instruction).
__device__ __forceinline__ void st_shared_b16_if(uint32_t addr, uint32_t v, bool p) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ne.b32 q, %2, 0;\n\t"
      "@q st.shared.b16 [%0], %1;\n\t}" ::"r"(addr), "h"(uint16_t(v)), "r"(int(p))
      : "memory");
}

// Writes one coefficient, given as two bf16 halves (hi | lo << 16), into the hi and lo
// tiles at (row, col) when `p` holds: two predicated stores, no branch (a branch around
// every entry's stores left the builder warps' tile writes several times slower).
__device__ __forceinline__ void put_if(uint8_t* hi_tile, uint8_t* lo_tile, int row, int col,
                                       uint32_t packed, bool p) {
  const uint32_t o = sw128_offset(row & (kBM - 1), col);
  st_shared_b16_if(smem_u32(hi_tile) + o, packed & 0xFFFFu, p);
  st_shared_b16_if(smem_u32(lo_tile) + o, packed >> 16, p);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ int64_t chunk_of(int64_t p, int64_t M, int n_c) {
  return (p * n_c) / M;
}

// Window [w0, w1) of sorted row p (round's sorted order), in sorted catalogue positions.
__device__ __forceinline__ void row_window(int64_t p, int64_t N, int64_t C, int n_c, int n_ec,
                                           int64_t& w0, int64_t& w1) {
  const int64_t c = chunk_of(p, N, n_c);
  w0 = chunk_start(c - n_ec < 0 ? 0 : c - n_ec, C, n_c);
  w1 = chunk_start(c + n_ec + 1 > n_c ? n_c : c + n_ec + 1, C, n_c);
}

// Epilogue of both band kernels: this thread's accumulator row (TMEM lane of the thread,
// ns columns) times `scale` into out row o -- stored when `write`, else added.  The rows
// are scattered (item ids or row ids of sorted positions), so each thread stages its row in
// pieces of W columns in shared memory (two buffers over the G tiles and B ring, free once
// the MMAs are done; rows padded by 16 B so that the float4 writes of 8 consecutive rows
// hit distinct banks) and hands each piece to the bulk-copy engine: full lines reach
// memory, and an add is done at L2 (the old values never come back to the SM).  One add
// per element per launch: deterministic.  `fin` must be uniform across the warp (the TMEM
// loads are warp-collective); rows with `live` false load but write nothing; `zero`
// (uniform across the CTA) writes zeros without reading TMEM.
__device__ __forceinline__ void epilogue_rows(uint8_t* stage, size_t avail, int t,
                                              uint32_t taddr, int ns, float scale, bool live,
                                              float* o, bool write, bool zero = false) {
  const int W = (ns % 128 == 0 && avail >= 2u * kBM * (128 * 4 + 16)) ? 128 : 64;
  const int stride = W * 4 + 16;
  for (int c0 = 0, piece = 0; c0 < ns; c0 += W, ++piece) {
    float* srow =
        reinterpret_cast<float*>(stage + size_t(piece & 1) * kBM * stride + size_t(t) * stride);
    bulk_wait_read<1>();  // this thread's copy out of that buffer (two pieces ago)
    for (int cc = 0; cc < W; cc += 32) {
      float v[32];
      if (zero) {  // no K slab: nothing was accumulated (CTA-uniform)
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] = 0.0f;
      } else {
        tmem_load32(taddr + uint32_t(c0 + cc), v);
      }
      float4* s4 = reinterpret_cast<float4*>(srow + cc);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        s4[u] = make_float4(scale * v[4 * u], scale * v[4 * u + 1], scale * v[4 * u + 2],
                            scale * v[4 * u + 3]);
    }
    if (live) {
      fence_proxy_async_smem();
      if (write)
        bulk_store(o + c0, srow, uint32_t(W) * 4u);
      else
        bulk_reduce_add_f32(o + c0, srow, uint32_t(W) * 4u);
      bulk_commit();
    }
  }
  bulk_wait_read<0>();  // the shared memory may go; the writes finish on their own
}

struct Args {
  int64_t N, C;
  int d, k, n_c, n_ec, r, ns, nb, Sp;
  const int32_t* px;        // [n_r][N] sorted row -> row (dY: py, sorted position -> item)
  const int2* kept;         // [n_r][N][k] (sorted position, p as bf16 hi | lo << 16)
  const int32_t* kept_off;  // [n_r][N][Sp] slice starts within the round's entries
  const float* dloss;       // [1]
  float* out;               // dX [N][d] (added into) or dY [C][d] (stored or added into)
  uint32_t* status;
  int write;                // dY: store (round 0, which covers every position), else add
  // dX with parts: one grid over (round, K split): blockIdx.z = round * ksplit + split;
  // each CTA stores its part to parts[z][row][:] (rows by id), added in z order after
  float* parts;
  int ksplit;
};

__device__ __forceinline__ void on_timeout(Ctl& c, uint32_t* status) {
  *reinterpret_cast<volatile int*>(&c.abort) = 1;
  raise_flag(status, RECE_DEVICE_TIMEOUT);
}

// One work item per CTA: 128 sorted rows of round r (K = the union of their windows);
// blockIdx.y picks the NS-wide slice of d.
__global__ void __launch_bounds__(kThreads, 1) k_bwd_dx_tc(const __grid_constant__ CUtensorMap tmB,
                                                        const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sbase = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* A_hi = sbase;
  uint8_t* A_lo = sbase + kAStages * kATile;
  uint8_t* Bs = sbase + 2 * kAStages * kATile;
  const uint32_t b_bytes = uint32_t(a.ns) * 128u;
  Ctl& ctl = *reinterpret_cast<Ctl*>(Bs + size_t(a.nb) * b_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, t = threadIdx.x;
  const int nb = a.nb;
  const int64_t N = a.N, C = a.C;
  const int r = a.parts ? int(blockIdx.z) / a.ksplit : a.r, n0 = blockIdx.y * a.ns;

  // the item's rows and its K range [lo, hi) in slabs of 64
  const int64_t m0 = int64_t(blockIdx.x) * kBM;
  int64_t lo = 0, hi = 0;
  {
    const int64_t last = (m0 + kBM - 1 < N - 1) ? m0 + kBM - 1 : N - 1;
    const int64_t cf = chunk_of(m0, N, a.n_c), cl = chunk_of(last, N, a.n_c);
    const int64_t k0 = chunk_start(cf - a.n_ec < 0 ? 0 : cf - a.n_ec, C, a.n_c);
    const int64_t k1 = chunk_start(cl + a.n_ec + 1 > a.n_c ? a.n_c : cl + a.n_ec + 1, C, a.n_c);
    if (k1 > k0) {
      lo = k0 >> 6;
      hi = (k1 + 63) >> 6;
    }
    if (a.parts && a.ksplit > 1) {  // this CTA's share of the slabs
      const int64_t n = hi - lo, sp = int64_t(blockIdx.z) % a.ksplit;
      hi = lo + n * (sp + 1) / a.ksplit;
      lo = lo + n * sp / a.ksplit;
    }
  }
  const int nK = int(hi - lo);

  if (t == 0) {
    for (int i = 0; i < nb; ++i) {
      mbar_init(&ctl.bfull[i], 1);
      mbar_init(&ctl.bempty[i], 1);
    }
    for (int i = 0; i < kAStages; ++i) {
      mbar_init(&ctl.afull[i], kBuilders / 32);  // one arrival per builder warp
      mbar_init(&ctl.aempty[i], 1);
    }
    mbar_init(&ctl.done, 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  const uint32_t tcols =
      a.ns <= 32 ? 32u : (a.ns <= 64 ? 64u : (a.ns <= 128 ? 128u : (a.ns <= 256 ? 256u : 512u)));
  if (warp == 4) {
    tmem_alloc(&ctl.tmem_base, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmB);
      int s = 0;
      for (; s < nK; ++s) {
        const int slot = s % nb;
        if (!mbar_wait(&ctl.bempty[slot], ((s / nb) & 1) ^ 1, &ctl.abort, kTimeoutNs)) {
          on_timeout(ctl, a.status);
          break;
        }
        mbar_arrive_expect_tx(&ctl.bfull[slot], b_bytes);
        for (int h = 0; h < a.ns; h += 64)  // boxes of 64 columns of d x 64 positions
          tma_load_3d(Bs + size_t(slot) * b_bytes + size_t(h) * 128, &tmB, &ctl.bfull[slot],
                      n0 + h, int((lo + s) * kBK), r);
      }
      for (int j = (s > nb ? s - nb : 0); j < s; ++j)  // every issued copy has landed
        mbar_wait_limit(&ctl.bfull[j % nb], (j / nb) & 1, kTimeoutNs);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // a slice of 512 columns is two MMAs of N = 256 into two accumulators
      const int nh = a.ns > 256 ? 2 : 1, nsh = a.ns / nh;
      const uint32_t idesc = idesc_bf16_f32_bmn(kBM, nsh);  // B (rows of d) MN-major
      for (int s = 0; s < nK; ++s) {
        const int as = s % kAStages, bs = s % nb;
        if (!mbar_wait(&ctl.afull[as], (s / kAStages) & 1, &ctl.abort, kTimeoutNs) ||
            !mbar_wait(&ctl.bfull[bs], (s / nb) & 1, &ctl.abort, kTimeoutNs)) {
          on_timeout(ctl, a.status);
          break;
        }
        tc_fence_after();
        const uint64_t dh = desc_k_plain(smem_u32(A_hi + as * kATile), 128u, 1024u);
        const uint64_t dl = desc_k_plain(smem_u32(A_lo + as * kATile), 128u, 1024u);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          for (int h = 0; h < nh; ++h) {
            // B: 64-column boxes 8 KB apart; 16 K rows of 128 B per MMA
            const uint64_t db =
                desc_mn_sw128(smem_u32(Bs + size_t(bs) * b_bytes + size_t(h) * nsh * 128),
                              8192u) + 128u * kk;
            const uint32_t acc = tmem + uint32_t(h * nsh);
            // K step kk: core matrices 2kk and 2kk + 1 along K, 256 B further
            mma_bf16(acc, dh + 16 * kk, db, idesc, (s | kk) != 0);
            mma_bf16(acc, dl + 16 * kk, db, idesc, 1);
          }
        }
        mma_commit(&ctl.aempty[as]);
        mma_commit(&ctl.bempty[bs]);
      }
      mma_commit(&ctl.done);
      mbar_wait_limit(&ctl.done, 0, kTimeoutNs);
    }
  } else {
    // ------------------------------------------------------------ builders
    const int64_t rN = int64_t(r) * N;
    constexpr int2 kNone = {0x7FFFFFFF, 0};  // past the last entry: beyond every slab
    // This thread's sorted row p = m0 + t.  Its round-r entries are grouped by slice in
    // ascending order, so the slabs consume them front to back, through a window of two
    // batches of 8 held in registers: cur = entries [base, base+8), nxt the 8 after, whose
    // loads are issued a batch ahead of their use.
    const int64_t p = m0 + t;
    const bool prow_ok = p < N;
    const int2* erow = a.kept + (rN + (prow_ok ? p : 0)) * a.k;
    int count = 0, e = 0, base = 0;
    int2 cur[8], nxt[8];
    if (prow_ok) {
      int64_t w0, w1;
      row_window(p, N, C, a.n_c, a.n_ec, w0, w1);
      const int S = w1 > w0 ? int((w1 - 1) >> 6) - int(w0 >> 6) + 1 : 0;
      const int32_t* offs = a.kept_off + (rN + p) * a.Sp;
      count = __ldg(offs + S);
      // the first entry at or past slab lo (a K split may start inside the window)
      const int64_t idx = lo - (w0 >> 6);
      e = idx <= 0 ? 0 : (idx >= S ? count : __ldg(offs + idx));
      base = e;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      cur[u] = e + u < count ? __ldg(erow + e + u) : kNone;
      nxt[u] = e + 8 + u < count ? __ldg(erow + e + 8 + u) : kNone;
    }

    for (int s = 0; s < nK; ++s) {
      const int as = s % kAStages;
      const bool waited = mbar_wait(&ctl.aempty[as], ((s / kAStages) & 1) ^ 1, &ctl.abort,
                                    kTimeoutNs);
      if (!waited) {  // each thread writes its own row only: no barrier to keep in step
        on_timeout(ctl, a.status);
        break;
      }
      uint8_t* th = A_hi + as * kATile;
      uint8_t* tl = A_lo + as * kATile;
      zero_row_plain(th, t);
      zero_row_plain(tl, t);
      const int64_t sig = lo + s;  // absolute slab
      const int slab_end = int((sig + 1) * kBK);
      while (e < count) {
        int used = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          // branch-free: the slot's two halves are stored under a predicate
          const bool in = base + u >= e && cur[u].x < slab_end;
          const int col = cur[u].x - int(sig * kBK);
          const bool put = in && col >= 0 && col < kBK;
          const uint32_t o = plain_offset(t, col & (kBK - 1));
          const uint32_t v = uint32_t(cur[u].y);
          st_shared_b16_if(smem_u32(th) + o, v & 0xFFFFu, put);
          st_shared_b16_if(smem_u32(tl) + o, v >> 16, put);
          used += in ? 1 : 0;
        }
        e += used;
        if (e < base + 8) break;  // the next entry belongs to a later slab
        // the batch is used up: the next one moves in, the one after is requested
#pragma unroll
        for (int u = 0; u < 8; ++u) cur[u] = nxt[u];
        base += 8;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          nxt[u] = base + 8 + u < count ? __ldg(erow + base + 8 + u) : kNone;
      }
      fence_proxy_async_smem();  // this thread's tile writes, visible to the MMA
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.afull[as]);
    }
    __syncwarp();

    // ------------------------------------------------------------ epilogue
    bool ok = mbar_wait(&ctl.done, 0, &ctl.abort, kTimeoutNs) && (nK > 0 || a.parts);
    ok = __all_sync(0xFFFFFFFFu, ok);
    const float scale = a.dloss[0] / float(N);  // G holds p; g = p * dloss / N
    tc_fence_after();
    const int64_t row = m0 + t;  // this thread's sorted row
    const bool live = row < N;
    const int64_t dst = live ? a.px[rN + row] : 0;
    // parts: every CTA stores its part (zeros when its split has no slab); else add
    float* o = a.parts ? a.parts + (int64_t(blockIdx.z) * N + dst) * a.d + n0
                       : a.out + dst * a.d + n0;
    if (ok)
      epilogue_rows(sbase, size_t(2 * kAStages) * kATile + size_t(nb) * b_bytes, t,
                    tmem + (uint32_t(warp * 32) << 16), a.ns, scale, live, o,
                    a.parts != nullptr, nK == 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// dY of step 6 on the tensor cores: per (round r, 128 sorted catalogue positions) the
// band product G_r[rows, positions]^T Xs_r[rows].  K = the rows whose windows cover the
// positions, in slabs of 64 rows.  Each builder thread owns one row of the slab and one
// 64-position half of the tile: it writes its row's kept entries there into the tile
// (items x rows, K-major: another thread's M row, so the tile is cleared, all builders
// meet at a named barrier, then fill it).  TMA streams the slab's 64 rows of the sorted
// copy Xs (MN-major B, as in the dX kernel), the MMAs and the epilogue are the dX kernel's; the epilogue adds into dY at the
// positions' item ids.  Round 0 writes every catalogue row (its tiles cover all positions),
// the later rounds add in round order, and the positives' terms are added after them (pair
// path): deterministic.
__global__ void __launch_bounds__(kThreads, 1) k_bwd_dy_tc(const __grid_constant__ CUtensorMap tmB,
                                                        const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* A_hi = base;
  uint8_t* A_lo = base + kAStages * kATile;
  uint8_t* Bs = base + 2 * kAStages * kATile;
  const uint32_t b_bytes = uint32_t(a.ns) * 128u;
  Ctl& ctl = *reinterpret_cast<Ctl*>(Bs + size_t(a.nb) * b_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, t = threadIdx.x;
  const int nb = a.nb;
  const int64_t N = a.N, C = a.C;
  const int r = a.r, n0 = blockIdx.y * a.ns;

  // the tile's positions and its K range [lo, hi) of 64-row slabs
  const int64_t q0 = int64_t(blockIdx.x) * kBM;
  int64_t k0 = 0, k1 = 0, lo = 0, hi = 0;
  {
    const int64_t last = (q0 + kBM - 1 < C - 1) ? q0 + kBM - 1 : C - 1;
    const int64_t cf = chunk_of(q0, C, a.n_c), cl = chunk_of(last, C, a.n_c);
    k0 = chunk_start(cf - a.n_ec < 0 ? 0 : cf - a.n_ec, N, a.n_c);
    k1 = chunk_start(cl + a.n_ec + 1 > a.n_c ? a.n_c : cl + a.n_ec + 1, N, a.n_c);
    if (k1 > k0) {
      lo = k0 >> 6;
      hi = (k1 + 63) >> 6;
    }
  }
  const int nK = int(hi - lo);

  if (t == 0) {
    for (int i = 0; i < nb; ++i) {
      mbar_init(&ctl.bfull[i], 1);
      mbar_init(&ctl.bempty[i], 1);
    }
    for (int i = 0; i < kAStages; ++i) {
      mbar_init(&ctl.afull[i], kBuilders / 32);
      mbar_init(&ctl.aempty[i], 1);
    }
    mbar_init(&ctl.done, 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  const uint32_t tcols =
      a.ns <= 32 ? 32u : (a.ns <= 64 ? 64u : (a.ns <= 128 ? 128u : (a.ns <= 256 ? 256u : 512u)));
  if (warp == 4) {
    tmem_alloc(&ctl.tmem_base, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmB);
      int s = 0;
      for (; s < nK; ++s) {
        const int slot = s % nb;
        if (!mbar_wait(&ctl.bempty[slot], ((s / nb) & 1) ^ 1, &ctl.abort, kTimeoutNs)) {
          on_timeout(ctl, a.status);
          break;
        }
        mbar_arrive_expect_tx(&ctl.bfull[slot], b_bytes);
        for (int h = 0; h < a.ns; h += 64)  // boxes of 64 columns of d x 64 positions
          tma_load_3d(Bs + size_t(slot) * b_bytes + size_t(h) * 128, &tmB, &ctl.bfull[slot],
                      n0 + h, int((lo + s) * kBK), r);
      }
      for (int j = (s > nb ? s - nb : 0); j < s; ++j)
        mbar_wait_limit(&ctl.bfull[j % nb], (j / nb) & 1, kTimeoutNs);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // a slice of 512 columns is two MMAs of N = 256 into two accumulators
      const int nh = a.ns > 256 ? 2 : 1, nsh = a.ns / nh;
      const uint32_t idesc = idesc_bf16_f32_bmn(kBM, nsh);  // B (rows of d) MN-major
      for (int s = 0; s < nK; ++s) {
        const int as = s % kAStages, bs = s % nb;
        if (!mbar_wait(&ctl.afull[as], (s / kAStages) & 1, &ctl.abort, kTimeoutNs) ||
            !mbar_wait(&ctl.bfull[bs], (s / nb) & 1, &ctl.abort, kTimeoutNs)) {
          on_timeout(ctl, a.status);
          break;
        }
        tc_fence_after();
        const uint64_t dh = desc_k_sw128(smem_u32(A_hi + as * kATile));
        const uint64_t dl = desc_k_sw128(smem_u32(A_lo + as * kATile));
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          for (int h = 0; h < nh; ++h) {
            // B: 64-column boxes 8 KB apart; 16 K rows of 128 B per MMA
            const uint64_t db =
                desc_mn_sw128(smem_u32(Bs + size_t(bs) * b_bytes + size_t(h) * nsh * 128),
                              8192u) + 128u * kk;
            const uint32_t acc = tmem + uint32_t(h * nsh);
            mma_bf16(acc, dh + 2 * kk, db, idesc, (s | kk) != 0);
            mma_bf16(acc, dl + 2 * kk, db, idesc, 1);
          }
        }
        mma_commit(&ctl.aempty[as]);
        mma_commit(&ctl.bempty[bs]);
      }
      mma_commit(&ctl.done);
      mbar_wait_limit(&ctl.done, 0, kTimeoutNs);
    }
  } else {
    // ------------------------------------------------------------ builders
    const int64_t rN = int64_t(r) * N;
    const int kc = t & (kBK - 1);  // this thread's row within a slab (the tile's K column)
    const int half = t >> 6;       // and its 64-position half of the tile
    const int64_t slice = (q0 >> 6) + half;
    // the entries of slab s's row in this half: [e0, e1) of its kept list, found a slab
    // ahead so that the offsets' load latency overlaps the previous slab
    // the window of this thread's row, tracked as the slabs advance (the row only grows):
    // the 64-bit divisions of the chunk arithmetic run when the row enters a new chunk,
    // not at every slab
    int64_t wc = -1, wc_hi = 0, sig0 = 0;  // the row's chunk, its end, its window's slab
    int wS = 0;                             // and the window's slab count
    auto set_chunk = [&](int64_t c) {
      wc = c;
      wc_hi = chunk_start(c + 1, N, a.n_c);
      const int64_t w0 = chunk_start(c - a.n_ec < 0 ? 0 : c - a.n_ec, C, a.n_c);
      const int64_t w1 = chunk_start(c + a.n_ec + 1 > a.n_c ? a.n_c : c + a.n_ec + 1, C, a.n_c);
      sig0 = w0 >> 6;
      wS = w1 > w0 ? int((w1 - 1) >> 6) - int(sig0) + 1 : 0;
    };
    auto entry_range = [&](int s2, int& e0, int& e1) {
      e0 = e1 = 0;
      const int64_t p = (lo + s2) * kBK + kc;  // sorted row (grows with s2)
      if (s2 >= nK || p < k0 || p >= k1 || p >= N) return;
      if (wc < 0) set_chunk(chunk_of(p, N, a.n_c));
      while (p >= wc_hi) set_chunk(wc + 1);
      const int64_t idx = slice - sig0;
      if (idx < 0 || idx >= wS) return;
      const int32_t* off = a.kept_off + (rN + p) * a.Sp;
      e0 = __ldg(off + idx);
      e1 = __ldg(off + idx + 1);
    };
    // Slab s's first kPre entries wait in registers, loaded while slab s - 1 was built
    // (its range known a slab earlier still), so the entry loads overlap the MMAs and
    // the clearing instead of following them; a longer run is loaded on the spot.
    constexpr int kPre = 16;
    auto slab_entries = [&](int s2) {
      return a.kept + (rN + (lo + s2) * kBK + kc) * a.k;
    };
    int a0, a1, b0, b1;  // entry ranges of slabs s and s + 1
    entry_range(0, a0, a1);
    entry_range(1, b0, b1);
    int2 pre[kPre];
    {
      const int2* ent = slab_entries(0);
#pragma unroll
      for (int u = 0; u < kPre; ++u)
        pre[u] = a0 + u < a1 ? __ldg(ent + a0 + u) : make_int2(0, 0);
    }
    bool ok = true;
    for (int s = 0; s < nK; ++s) {
      const int as = s % kAStages;
      // every builder runs every slab to the named barriers, also after a timeout
      if (ok && !mbar_wait(&ctl.aempty[as], ((s / kAStages) & 1) ^ 1, &ctl.abort, kTimeoutNs)) {
        on_timeout(ctl, a.status);
        ok = false;
      }
      uint8_t* th = A_hi + as * kATile;
      uint8_t* tl = A_lo + as * kATile;
      if (ok) {
        zero_row(th, t);
        zero_row(tl, t);
      }
      named_barrier(1, kBuilders);  // the whole tile is clear before anyone fills it
      int c0, c1;
      entry_range(s + 2, c0, c1);
      if (ok && a1 > a0) {
#pragma unroll
        for (int u = 0; u < kPre; ++u)
          put_if(th, tl, int(pre[u].x - q0), kc, uint32_t(pre[u].y), a0 + u < a1);
        const int2* ent = slab_entries(s);
        for (int e = a0 + kPre; e < a1; e += 8) {  // the rest, eight loads in flight
          int2 en[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) en[u] = e + u < a1 ? __ldg(ent + e + u) : make_int2(0, 0);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            put_if(th, tl, int(en[u].x - q0), kc, uint32_t(en[u].y), e + u < a1);
        }
      }
      {  // slab s + 1's first entries
        const int2* ent = slab_entries(s + 1);
#pragma unroll
        for (int u = 0; u < kPre; ++u)
          pre[u] = b0 + u < b1 ? __ldg(ent + b0 + u) : make_int2(0, 0);
      }
      a0 = b0;
      a1 = b1;
      b0 = c0;
      b1 = c1;
      fence_proxy_async_smem();  // this thread's tile writes, visible to the MMA
      named_barrier(1, kBuilders);  // nobody clears the next tile into this one's readers
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&ctl.afull[as]);
    }
    __syncwarp();

    // ------------------------------------------------------------ epilogue
    bool fin = ok && mbar_wait(&ctl.done, 0, &ctl.abort, kTimeoutNs) && nK > 0;
    fin = __all_sync(0xFFFFFFFFu, fin);
    tc_fence_after();
    const float scale = a.dloss[0] / float(N);  // G holds p; g = p * dloss / N
    const int64_t q = q0 + t;                   // this thread's sorted position
    const bool live = q < C;
    const int64_t dst = live ? a.px[int64_t(r) * C + q] : 0;
    if (fin)
      epilogue_rows(base, size_t(2 * kAStages) * kATile + size_t(nb) * b_bytes, t,
                    tmem + (uint32_t(warp * 32) << 16), a.ns, scale, live,
                    a.out + dst * a.d + n0, a.write);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// Persistent dY (slices of 256 columns of d): one CTA per SM loops over work items
// (128 sorted catalogue positions x one slice of d), so the fixed cost of a CTA -- barrier
// set-up, TMEM allocation, the first entry loads, the epilogue's tail -- is paid once per
// SM instead of once per item, and one item's epilogue overlaps the next one's tiles and
// MMAs: TMEM holds two accumulators (item parity), four epilogue warps drain one while the
// MMAs fill the other, and stage their rows in a shared-memory area of their own.  The
// builders, the TMA producer and the MMA issuer run the items' slabs through the rings
// back to back.  Per item the computation is k_bwd_dy_tc's (each dY row written or added
// by one CTA per launch, K in a fixed order): deterministic.
constexpr int kPEpi = 128;                       // epilogue threads (warps 6-9)
constexpr int kPThreads = kBuilders + 64 + kPEpi;
constexpr int kPW = 32;                          // epilogue piece: 32 columns a row
constexpr int kPStride = kPW * 4 + 16;           // staged row piece, padded by 16 B

struct CtlP {
  uint64_t bfull[kMaxBStages], bempty[kMaxBStages];
  uint64_t afull[kAStages], aempty[kAStages];
  uint64_t accfull[2], accempty[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
};

__host__ __device__ constexpr size_t smem_bytes_p(int nb, int ns) {
  return 1024 + size_t(2 * kAStages) * kATile + size_t(nb) * ns * 128 +
         size_t(2) * kPEpi * kPStride + sizeof(CtlP);
}

struct DyItem {
  int64_t q0, k0, k1, lo;
  int nK, n0;
};
__device__ __forceinline__ DyItem dy_item(int64_t it, int slices, int ns, int64_t N,
                                          int64_t C, int n_c, int n_ec) {
  DyItem g;
  g.q0 = (it / slices) * kBM;
  g.n0 = int(it % slices) * ns;
  const int64_t last = (g.q0 + kBM - 1 < C - 1) ? g.q0 + kBM - 1 : C - 1;
  const int64_t cf = chunk_of(g.q0, C, n_c), cl = chunk_of(last, C, n_c);
  g.k0 = chunk_start(cf - n_ec < 0 ? 0 : cf - n_ec, N, n_c);
  g.k1 = chunk_start(cl + n_ec + 1 > n_c ? n_c : cl + n_ec + 1, N, n_c);
  g.lo = 0;
  g.nK = 0;
  if (g.k1 > g.k0) {
    g.lo = g.k0 >> 6;
    g.nK = int(((g.k1 + 63) >> 6) - g.lo);
  }
  return g;
}

__device__ __forceinline__ void on_timeout_p(CtlP& c, uint32_t* status) {
  *reinterpret_cast<volatile int*>(&c.abort) = 1;
  raise_flag(status, RECE_DEVICE_TIMEOUT);
}

__global__ void __launch_bounds__(kPThreads, 1) k_bwd_dy_tc_p(const __grid_constant__ CUtensorMap tmB,
                                                          const Args a, int64_t items,
                                                          int slices) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* A_hi = base;
  uint8_t* A_lo = base + kAStages * kATile;
  uint8_t* Bs = base + 2 * kAStages * kATile;
  const uint32_t b_bytes = uint32_t(a.ns) * 128u;
  uint8_t* stage = Bs + size_t(a.nb) * b_bytes;
  CtlP& ctl = *reinterpret_cast<CtlP*>(stage + size_t(2) * kPEpi * kPStride);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, t = threadIdx.x;
  const int nb = a.nb, ns = a.ns;
  const int64_t N = a.N, C = a.C;
  const int r = a.r;

  if (t == 0) {
    for (int i = 0; i < nb; ++i) {
      mbar_init(&ctl.bfull[i], 1);
      mbar_init(&ctl.bempty[i], 1);
    }
    for (int i = 0; i < kAStages; ++i) {
      mbar_init(&ctl.afull[i], kBuilders / 32);
      mbar_init(&ctl.aempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.accfull[i], 1);
      mbar_init(&ctl.accempty[i], kPEpi / 32);
    }
    mbar_init(&ctl.done, 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  const uint32_t tcols = ns <= 32 ? 64u : (ns <= 64 ? 128u : (ns <= 128 ? 256u : 512u));
  if (warp == 4) {
    tmem_alloc(&ctl.tmem_base, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmB);
      uint32_t sg = 0;  // slabs issued so far (all items)
      bool ok = true;
      for (int64_t it = blockIdx.x; it < items && ok; it += gridDim.x) {
        const DyItem g = dy_item(it, slices, ns, N, C, a.n_c, a.n_ec);
        for (int s = 0; s < g.nK; ++s, ++sg) {
          const int slot = int(sg % uint32_t(nb));
          if (!mbar_wait(&ctl.bempty[slot], ((sg / nb) & 1u) ^ 1u, &ctl.abort, kTimeoutNs)) {
            on_timeout_p(ctl, a.status);
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&ctl.bfull[slot], b_bytes);
          for (int h = 0; h < ns; h += 64)  // boxes of 64 columns of d x 64 rows
            tma_load_3d(Bs + size_t(slot) * b_bytes + size_t(h) * 128, &tmB, &ctl.bfull[slot],
                        g.n0 + h, int((g.lo + s) * kBK), r);
        }
      }
      for (uint32_t j = (sg > uint32_t(nb) ? sg - nb : 0); j < sg; ++j)
        mbar_wait_limit(&ctl.bfull[j % nb], (j / nb) & 1u, kTimeoutNs);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32_bmn(kBM, ns);  // B (rows of d) MN-major
      uint32_t sg = 0, il = 0;  // slabs consumed, items begun by this CTA
      bool ok = true;
      for (int64_t it = blockIdx.x; it < items && ok; it += gridDim.x, ++il) {
        const DyItem g = dy_item(it, slices, ns, N, C, a.n_c, a.n_ec);
        const int acc = int(il & 1u);
        if (!mbar_wait(&ctl.accempty[acc], ((il >> 1) & 1u) ^ 1u, &ctl.abort, kTimeoutNs)) {
          on_timeout_p(ctl, a.status);
          break;
        }
        tc_fence_after();
        const uint32_t d_acc = tmem + uint32_t(acc * ns);
        for (int s = 0; s < g.nK; ++s, ++sg) {
          const int as = int(sg % kAStages), bs = int(sg % uint32_t(nb));
          if (!mbar_wait(&ctl.afull[as], (sg / kAStages) & 1u, &ctl.abort, kTimeoutNs) ||
              !mbar_wait(&ctl.bfull[bs], (sg / nb) & 1u, &ctl.abort, kTimeoutNs)) {
            on_timeout_p(ctl, a.status);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dh = desc_k_sw128(smem_u32(A_hi + as * kATile));
          const uint64_t dl = desc_k_sw128(smem_u32(A_lo + as * kATile));
          const uint64_t db0 = desc_mn_sw128(smem_u32(Bs + size_t(bs) * b_bytes), 8192u);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t db = db0 + 128u * kk;  // 16 K rows of 128 B per MMA
            mma_bf16(d_acc, dh + 2 * kk, db, idesc, (s | kk) != 0);
            mma_bf16(d_acc, dl + 2 * kk, db, idesc, 1);
          }
          mma_commit(&ctl.aempty[as]);
          mma_commit(&ctl.bempty[bs]);
        }
        if (!ok) break;
        mma_commit(&ctl.accfull[acc]);
      }
      mma_commit(&ctl.done);
      mbar_wait_limit(&ctl.done, 0, kTimeoutNs);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ builders
    // As in k_bwd_dy_tc: thread t owns row kc = t % 64 of every slab and the 64-position
    // half t / 64 of the tile; it clears its row of both halves' tiles, all builders meet,
    // then each writes its row's kept entries that fall in its half.  Every builder runs
    // every item and slab to the named barriers, also after a timeout.
    const int64_t rN = int64_t(r) * N;
    const int kc = t & (kBK - 1);
    const int half = t >> 6;
    uint32_t sg = 0;
    bool ok = true;
    for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
      const DyItem g = dy_item(it, slices, ns, N, C, a.n_c, a.n_ec);
      const int64_t slice = (g.q0 >> 6) + half;
      int64_t wc = -1, wc_hi = 0, sig0 = 0;
      int wS = 0;
      auto set_chunk = [&](int64_t c) {
        wc = c;
        wc_hi = chunk_start(c + 1, N, a.n_c);
        const int64_t w0 = chunk_start(c - a.n_ec < 0 ? 0 : c - a.n_ec, C, a.n_c);
        const int64_t w1 =
            chunk_start(c + a.n_ec + 1 > a.n_c ? a.n_c : c + a.n_ec + 1, C, a.n_c);
        sig0 = w0 >> 6;
        wS = w1 > w0 ? int((w1 - 1) >> 6) - int(sig0) + 1 : 0;
      };
      auto entry_range = [&](int s2, int& e0, int& e1) {
        e0 = e1 = 0;
        const int64_t p = (g.lo + s2) * kBK + kc;  // sorted row (grows with s2)
        if (s2 >= g.nK || p < g.k0 || p >= g.k1 || p >= N) return;
        if (wc < 0) set_chunk(chunk_of(p, N, a.n_c));
        while (p >= wc_hi) set_chunk(wc + 1);
        const int64_t idx = slice - sig0;
        if (idx < 0 || idx >= wS) return;
        const int32_t* off = a.kept_off + (rN + p) * a.Sp;
        e0 = __ldg(off + idx);
        e1 = __ldg(off + idx + 1);
      };
      constexpr int kPre = 8;  // entries prefetched per (row, half); more take the loop below
      auto slab_entries = [&](int s2) { return a.kept + (rN + (g.lo + s2) * kBK + kc) * a.k; };
      int a0, a1, b0, b1;
      entry_range(0, a0, a1);
      entry_range(1, b0, b1);
      int2 pre[kPre];
      {
        const int2* ent = slab_entries(0);
#pragma unroll
        for (int u = 0; u < kPre; ++u)
          pre[u] = a0 + u < a1 ? __ldg(ent + a0 + u) : make_int2(0, 0);
      }
      for (int s = 0; s < g.nK; ++s, ++sg) {
        const int as = int(sg % kAStages);
        if (ok && !mbar_wait(&ctl.aempty[as], ((sg / kAStages) & 1u) ^ 1u, &ctl.abort,
                             kTimeoutNs)) {
          on_timeout_p(ctl, a.status);
          ok = false;
        }
        uint8_t* th = A_hi + as * kATile;
        uint8_t* tl = A_lo + as * kATile;
        if (ok) {
          zero_row(th, t);
          zero_row(tl, t);
        }
        named_barrier(1, kBuilders);  // the whole tile is clear before anyone fills it
        int c0, c1;
        entry_range(s + 2, c0, c1);
        if (ok && a1 > a0) {
#pragma unroll
          for (int u = 0; u < kPre; ++u)
            put_if(th, tl, int(pre[u].x - g.q0), kc, uint32_t(pre[u].y), a0 + u < a1);
          const int2* ent = slab_entries(s);
          for (int e = a0 + kPre; e < a1; e += 8) {
            int2 en[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) en[u] = e + u < a1 ? __ldg(ent + e + u) : make_int2(0, 0);
#pragma unroll
            for (int u = 0; u < 8; ++u)
              put_if(th, tl, int(en[u].x - g.q0), kc, uint32_t(en[u].y), e + u < a1);
          }
        }
        {
          const int2* ent = slab_entries(s + 1);
#pragma unroll
          for (int u = 0; u < kPre; ++u)
            pre[u] = b0 + u < b1 ? __ldg(ent + b0 + u) : make_int2(0, 0);
        }
        a0 = b0;
        a1 = b1;
        b0 = c0;
        b1 = c1;
        fence_proxy_async_smem();
        named_barrier(1, kBuilders);  // nobody clears the next tile into this one's readers
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&ctl.afull[as]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int row = ((warp & 3) << 5) + lane;  // this thread's TMEM lane (tile row)
    float* const buf0 = reinterpret_cast<float*>(stage + size_t(row) * kPStride);
    float* const buf1 = reinterpret_cast<float*>(stage + size_t(kPEpi + row) * kPStride);
    const float scale = a.dloss[0] / float(N);  // G holds p; g = p * dloss / N
    uint32_t il = 0, piece = 0;
    bool ok = true;
    for (int64_t it = blockIdx.x; it < items; it += gridDim.x, ++il) {
      const DyItem g = dy_item(it, slices, ns, N, C, a.n_c, a.n_ec);
      const int acc = int(il & 1u);
      bool fin = ok && mbar_wait(&ctl.accfull[acc], (il >> 1) & 1u, &ctl.abort, kTimeoutNs);
      fin = __all_sync(0xFFFFFFFFu, fin);
      if (!fin) {
        if (ok) on_timeout_p(ctl, a.status);
        ok = false;
        continue;
      }
      tc_fence_after();
      const int64_t q = g.q0 + row;
      const bool live = q < C;
      const int64_t dst = live ? a.px[int64_t(r) * C + q] : -1;
      const uint32_t taddr = tmem + (uint32_t((warp & 3) * 32) << 16) + uint32_t(acc * ns);
      // Each piece of 32 columns goes through the warp's staging rows and out as whole
      // 128-byte row segments: lanes 8j..8j+7 write 16 B each of one row, four rows a store
      // (the rows are items, scattered); the warp's rows' destinations come by shuffle.
      for (int c0 = 0; c0 < ns; c0 += kPW, ++piece) {
        float* srow = (piece & 1u) ? buf1 : buf0;
        float v[32];
        if (g.nK == 0) {  // no rows cover the item: nothing accumulated (uniform)
#pragma unroll
          for (int u = 0; u < 32; ++u) v[u] = 0.0f;
        } else {
          tmem_load32(taddr + uint32_t(c0), v);
        }
        float4* s4 = reinterpret_cast<float4*>(srow);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          s4[u] = make_float4(scale * v[4 * u], scale * v[4 * u + 1], scale * v[4 * u + 2],
                              scale * v[4 * u + 3]);
        __syncwarp();
        const uint8_t* wbase = reinterpret_cast<const uint8_t*>(srow) - size_t(lane) * kPStride;
#pragma unroll
        for (int it4 = 0; it4 < 8; ++it4) {
          const int rr = 4 * it4 + (lane >> 3), ch = lane & 7;
          const int64_t drow = __shfl_sync(0xFFFFFFFFu, dst, rr);
          const float4 x = *reinterpret_cast<const float4*>(wbase + size_t(rr) * kPStride + ch * 16);
          if (drow >= 0) {
            float4* out = reinterpret_cast<float4*>(a.out + drow * a.d + g.n0 + c0) + ch;
            if (a.write) {
              *out = x;
            } else {  // later rounds add (one writer per element and launch: a fixed order)
              const float4 y = *out;
              *out = make_float4(y.x + x.x, y.y + x.y, y.z + x.z, y.w + x.w);
            }
          }
        }
      }
      tc_fence_before();  // the accumulator's reads are done: the MMAs may refill it
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.accempty[acc]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// One warp per row: the positive's coefficient g_iz and dX_i = g_iz y_z (written, not
// added: the rounds add after it).
template <typename T>
__global__ void __launch_bounds__(256) k_bwd_pos(const T* __restrict__ Y,
                                                 const int32_t* __restrict__ targets,
                                                 const float* __restrict__ lse,
                                                 const float* __restrict__ pos_logit,
                                                 const float* __restrict__ dloss, int64_t N,
                                                 int64_t C, int d, float* __restrict__ dX) {
  const int lane = threadIdx.x & 31;
  const int64_t i = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (i >= N) return;
  const int32_t z = targets[i];
  const bool z_ok = z >= 0 && z < C;
  float g = 0.0f;
  if (z_ok) g = (expf(pos_logit[i] - lse[i]) - 1.0f) * (dloss[0] / float(N));
  const T* y = Y + (z_ok ? int64_t(z) : 0) * d;
  for (int t = 8 * lane; t < d; t += 256) {
    float v[8];
    load8(y + t, v);
    float4* o = reinterpret_cast<float4*>(dX + i * d + t);
    o[0] = make_float4(g * v[0], g * v[1], g * v[2], g * v[3]);
    o[1] = make_float4(g * v[4], g * v[5], g * v[6], g * v[7]);
  }
}

}  // namespace

// Band-product geometry for d: CTA slices of ns <= 512 columns (two TMEM accumulators
// past 256) and a TMA ring as deep as lets two CTAs share an SM (at least two slabs), or,
// where two cannot share one (ns >= 256), as deep as one CTA's shared memory allows (at
// the 4M-item workload, d = 256: dY 4.16 -> 3.76 ms, its CTAs' few slabs all in flight).
struct BandGeometry {
  int ns, slices, nb;
  size_t smem;
  uint32_t tcols;
};
BandGeometry band_geometry(int d) {
  BandGeometry g;
  g.ns = d;
  if (g.ns > 256)
    g.ns = (d % 512 == 0) ? 512
                          : (d % 256 == 0 ? 256 : (d % 192 == 0 ? 192 : (d % 128 == 0 ? 128 : 64)));
  g.slices = d / g.ns;
  int nb = int((110 * 1024 - 2 * kAStages * kATile - 1024 - sizeof(Ctl)) / (size_t(g.ns) * 128));
  if (nb < 2)  // two CTAs cannot share an SM anyway: one CTA takes the SM's shared memory
    nb = int((227 * 1024 - 2 * kAStages * kATile - 1024 - sizeof(Ctl)) / (size_t(g.ns) * 128));
  g.nb = nb > kMaxBStages ? kMaxBStages : (nb < 2 ? 2 : nb);
  g.smem = smem_bytes(g.nb, g.ns);
  g.tcols = g.ns <= 32 ? 32u : (g.ns <= 64 ? 64u : (g.ns <= 128 ? 128u : (g.ns <= 256 ? 256u : 512u)));
  return g;
}

template <typename T>
cudaError_t launch_dx_tc(const rece_plan_s& p, const T* Y, const int32_t* targets,
                         const float* lse, const float* dloss, char* ws, float* dX,
                         uint32_t* status, cudaStream_t st) {
  const auto& c = p.cfg;
  const Layout& L = p.lay;
  if (c.N == 0) return cudaSuccess;
  const BandGeometry g = band_geometry(c.d);
  const int ns = g.ns, slices = g.slices, nb = g.nb;
  const size_t smem = g.smem;

  Args a{};
  a.N = c.N;
  a.C = c.C;
  a.d = c.d;
  a.k = c.k;
  a.n_c = c.n_c;
  a.n_ec = c.n_ec;
  a.ns = ns;
  a.nb = nb;
  a.Sp = p.kept_slices + 1;
  a.px = reinterpret_cast<const int32_t*>(ws + L.px);
  a.kept = reinterpret_cast<const int2*>(ws + L.kept);
  a.kept_off = reinterpret_cast<const int32_t*>(ws + L.kept_off);
  a.dloss = dloss;
  a.status = status;
  a.out = dX;

  k_bwd_pos<T><<<unsigned(ceil_div(c.N, 8)), 256, 0, st>>>(
      Y, targets, lse, reinterpret_cast<const float*>(ws + L.pos_logit), dloss, c.N, c.C, c.d,
      dX);
  count_launches(1);
  RECE_TRY(cudaGetLastError());
  RECE_TRY(cudaFuncSetAttribute(k_bwd_dx_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(smem)));
  CUtensorMap tm;  // the sorted rows of Y of every round, read MN-major
  RECE_TRY(make_tmap_bf16_3d(&tm, ws + L.ys, uint64_t(c.d), uint64_t(c.C), uint64_t(c.n_r),
                             uint32_t(kBK)));
  if (p.dx_split > 0) {
    // one grid over (round, K split), parts stored, then added into dX in order
    a.parts = reinterpret_cast<float*>(ws + L.dx_parts);
    a.ksplit = p.dx_split;
    const int nz = c.n_r * p.dx_split;
    k_bwd_dx_tc<<<dim3(unsigned(ceil_div(c.N, kBM)), unsigned(slices), unsigned(nz)), kThreads,
                  smem, st>>>(tm, a);
    count_launches(1);
    RECE_TRY(cudaGetLastError());
    return launch_add_parts(a.parts, c.N * int64_t(c.d), nz, dX, st);
  }
  for (int r = 0; r < c.n_r; ++r) {  // rounds in order, each adding into dX
    a.r = r;
    k_bwd_dx_tc<<<dim3(unsigned(ceil_div(c.N, kBM)), unsigned(slices)), kThreads, smem, st>>>(
        tm, a);
    count_launches(1);
    RECE_TRY(cudaGetLastError());
  }
  return cudaSuccess;
}

// How the dX band products cover the rounds.  Per-round launches (0) leave the last wave
// of each launch part-empty when a round has few work items; one launch over (round, K
// split) with S splits of every work item's window (S >= 1) fills the waves at the price
// of n_r S parts of dX written and summed in order.  Chosen from the wave counts, in units
// of one whole-window work item; a split keeps at least 8 slabs of the narrowest window.
int dx_tc_split(const rece_plan_s& p) {
  const auto& c = p.cfg;
  if (c.N == 0 || c.n_c < 1) return 0;
  const BandGeometry g = band_geometry(c.d);
  int per_sm = int((228 * 1024) / (g.smem + 1024));
  if (per_sm > int(512 / g.tcols)) per_sm = int(512 / g.tcols);
  if (per_sm < 1) per_sm = 1;
  const double slots = double(sm_count()) * per_sm;
  const double items = double(ceil_div(c.N, kBM)) * g.slices;  // per round
  double best = c.n_r * std::ceil(items / slots);
  int pick = 0;
  const int64_t edge_chunks = c.n_ec + 1 < c.n_c ? c.n_ec + 1 : c.n_c;
  const int64_t min_slabs = (c.C * edge_chunks / c.n_c) / kBK;
  for (int S = 1; S <= 4; ++S) {
    if (S > 1 && min_slabs / S < 8) break;
    const double cost = std::ceil(c.n_r * items * S / slots) / S;
    if (cost < 0.9 * best) {
      best = cost;
      pick = S;
    }
  }
  return pick;
}

// The window terms of dY: round 0 stores them (its tiles cover every catalogue position),
// the later rounds add.
cudaError_t launch_dy_tc(const rece_plan_s& p, const float* dloss, char* ws, float* dY,
                         uint32_t* status, cudaStream_t st) {
  const auto& c = p.cfg;
  const Layout& L = p.lay;
  if (c.N == 0) return cudaSuccess;
  const BandGeometry g = band_geometry(c.d);
  const int ns = g.ns, slices = g.slices, nb = g.nb;
  const size_t smem = g.smem;
  Args a{};
  a.N = c.N;
  a.C = c.C;
  a.d = c.d;
  a.k = c.k;
  a.n_c = c.n_c;
  a.n_ec = c.n_ec;
  a.ns = ns;
  a.nb = nb;
  a.Sp = p.kept_slices + 1;
  a.px = reinterpret_cast<const int32_t*>(ws + L.py);
  a.kept = reinterpret_cast<const int2*>(ws + L.kept);
  a.kept_off = reinterpret_cast<const int32_t*>(ws + L.kept_off);
  a.dloss = dloss;
  a.status = status;
  a.out = dY;
  CUtensorMap tm;  // the sorted rows of X of every round, read MN-major
  RECE_TRY(make_tmap_bf16_3d(&tm, ws + L.xs, uint64_t(c.d), uint64_t(c.N), uint64_t(c.n_r),
                             uint32_t(kBK)));
  if (ns == 256) {
    // persistent: a CTA per SM over (position tile, slice) items, the B ring as deep as
    // the shared memory left beside the G stages and the epilogue's staging allows (at
    // the 4M-item workload, d = 256: 3.76 -> 2.79 ms; at d = 128 two CTAs of the
    // per-item kernel share an SM and their builders outrun one persistent CTA's:
    // 1.35 -> 2.01 ms there, so narrower slices keep k_bwd_dy_tc)
    const size_t fixed = smem_bytes_p(0, ns);
    int nbp = int((227 * 1024 - fixed) / (size_t(ns) * 128));
    nbp = nbp > kMaxBStages ? kMaxBStages : nbp;
    if (nbp >= 2) {
      a.nb = nbp;
      const size_t smem_p = smem_bytes_p(nbp, ns);
      RECE_TRY(cudaFuncSetAttribute(k_bwd_dy_tc_p, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    int(smem_p)));
      const int64_t items = ceil_div(c.C, kBM) * slices;
      const int grid = int(items < sm_count() ? items : sm_count());
      for (int r = 0; r < c.n_r; ++r) {
        a.r = r;
        a.write = r == 0;
        k_bwd_dy_tc_p<<<grid, kPThreads, smem_p, st>>>(tm, a, items, slices);
        count_launches(1);
        RECE_TRY(cudaGetLastError());
      }
      return cudaSuccess;
    }
  }
  RECE_TRY(cudaFuncSetAttribute(k_bwd_dy_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(smem)));
  for (int r = 0; r < c.n_r; ++r) {
    a.r = r;
    a.write = r == 0;
    k_bwd_dy_tc<<<dim3(unsigned(ceil_div(c.C, kBM)), unsigned(slices)), kThreads, smem, st>>>(
        tm, a);
    count_launches(1);
    RECE_TRY(cudaGetLastError());
  }
  return cudaSuccess;
}

template cudaError_t launch_dx_tc<__nv_bfloat16>(const rece_plan_s&, const __nv_bfloat16*,
                                                 const int32_t*, const float*, const float*,
                                                 char*, float*, uint32_t*, cudaStream_t);

}  // namespace rece
