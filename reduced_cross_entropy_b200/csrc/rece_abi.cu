// rece_abi.cu -- the C ABI declared in include/rece.h: plan validation, workspace
// layout and the launch sequence of every entry point.  No device memory is allocated
// here: every device buffer, the workspace included, belongs to the caller.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <new>

#include "common.cuh"
#include "plan.h"
#include "tc.h"

namespace rece {
size_t select_fma_smem_bytes(int G, int d, int64_t w_max);
int merge_pow2(int n_r, int k);

namespace {
std::atomic<uint64_t> g_launches{0};
}
void count_launches(int n) { g_launches.fetch_add(uint64_t(n), std::memory_order_relaxed); }
void set_last_error(const char* msg);
}  // namespace rece

using namespace rece;

namespace {

constexpr size_t kMaxSmem = 227 * 1024;
constexpr int64_t kInt32Max = 2147483647;

thread_local char g_last_error[256] = "";

rece_status_t fail(rece_status_t s, const char* msg) {
  snprintf(g_last_error, sizeof(g_last_error), "%s", msg);
  return s;
}

rece_status_t cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorName(e),
           cudaGetErrorString(e));
  return RECE_ERR_CUDA;
}

#define RECE_CUDA(call, where)                   \
  do {                                           \
    cudaError_t e_ = (call);                     \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

int64_t window_len(int64_t c, int64_t C, int64_t n_c, int64_t n_ec) {
  const int64_t lo = c - n_ec < 0 ? 0 : c - n_ec;
  const int64_t hi = c + n_ec + 1 > n_c ? n_c : c + n_ec + 1;
  return chunk_start(hi, C, n_c) - chunk_start(lo, C, n_c);
}

// The backward's (item, row) pair arrays from offset `off` on.
void layout_pairs(rece_plan_s& p, size_t& off) {
  Layout& L = p.lay;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t E = size_t(p.entries);
  L.e_key = take(sizeof(int32_t) * E);
  L.e_g = take(sizeof(float) * E);
  L.e_perm_a = take(sizeof(int32_t) * E);
  L.e_perm_b = take(sizeof(int32_t) * E);
  L.e_sorted_key = take(sizeof(int32_t) * E);
  L.e_key_b = take(sizeof(int32_t) * E);
  if (p.carry_g) {
    L.e_sorted_g = take(sizeof(float) * E);
    L.e_g_b = take(sizeof(float) * E);
  }
  L.e_item_start = take(sizeof(int32_t) * (size_t(p.cfg.C) + 1));
  L.e_scratch = take(sort_scratch_bytes(p.entries, p.item_pass_bits));
  L.e_long = take(sizeof(int32_t) * (E / kLongRunPairs + 2));
}

// Item-sort geometry of the backward's pairs (keys 0..C: C marks an empty slot).  Digits
// of at most 9 bits: a 2048-pair tile scatters into at most 512 runs, so its writes stay
// in runs of several pairs; wider digits leave about one pair per run (measured: 9 ps per
// pair and pass at 9 bits, 23 at 10, 45 at 11-12), and a third pass costs less than that.
constexpr int kPairDigitBits = 9;
void set_pair_sort(rece_plan_s& p) {
  const auto& c = p.cfg;
  p.item_bits = bits_for(c.C + 1);
  p.item_passes = int32_t((p.item_bits + kPairDigitBits - 1) / kPairDigitBits);
  if (p.item_passes < 1) p.item_passes = 1;
  p.item_pass_bits = (p.item_bits + p.item_passes - 1) / p.item_passes;
  p.entries = c.N * (int64_t(c.k) + 1);
  p.carry_g = p.entries * int64_t(sizeof(float)) > (int64_t(32) << 20);
}

// All-negatives mode: what the backward reads stays from rece_bucketize_sort on (sorted
// copies, orders, chunk tables, positives' sorted positions, lse by
// round); the forward's scratch and the positives' pair arrays share the rest.
void build_layout_all_neg(rece_plan_s& p) {
  const auto& c = p.cfg;
  Layout& L = p.lay;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  L.status = take(4 * sizeof(uint32_t));
  const size_t nb_stride = (size_t(1) << p.bucket_bits) + 1;
  const size_t nr = size_t(c.n_r);
  L.px = take(sizeof(int32_t) * nr * c.N);
  L.py = take(sizeof(int32_t) * nr * c.C);
  if (p.window_tc) {  // the tcgen05 kernels' sorted copies (the CUDA-core ones read X, Y)
    L.xs = take(sizeof(uint16_t) * nr * c.N * c.d);
    L.ys = take(sizeof(uint16_t) * nr * c.C * c.d);
  }
  L.itemc = take(sizeof(int32_t) * nr * nr * c.C);
  L.rowc = take(sizeof(int32_t) * nr * nr * c.N);
  L.pz = take(sizeof(int32_t) * nr * c.N);
  L.lse_sorted = take(sizeof(float) * nr * c.N);
  const size_t region = off;
  L.bx = take(sizeof(int32_t) * nr * c.N);
  L.by = take(sizeof(int32_t) * nr * c.C);
  L.bstart_x = take(sizeof(int32_t) * nr * nb_stride);
  L.bstart_y = take(sizeof(int32_t) * nr * nb_stride);
  L.sort_scratch = take(nr * (sort_hist_bytes(c.N, p.bucket_bits) +
                              sort_hist_bytes(c.C, p.bucket_bits)));
  L.inv_x = take(sizeof(int32_t) * nr * c.N);
  L.inv_y = take(sizeof(int32_t) * nr * c.C);
  L.ms = take(sizeof(float) * 2 * nr * c.N);
  L.row_loss_tmp = take(sizeof(float) * c.N);
  L.fwd_end = off;
  off = region;
  rece_plan_s& q = *p.pos_plan;
  q.lay.status = L.status;
  layout_pairs(q, off);
  if (p.window_tc) L.dx_parts = take(sizeof(float) * nr * c.N * c.d);  // each round's part of dX
  L.bwd_end = off;
  L.total = L.fwd_end > L.bwd_end ? L.fwd_end : L.bwd_end;
}

void build_layout(rece_plan_s& p) {
  if (p.all_neg) {
    build_layout_all_neg(p);
    return;
  }
  const auto& c = p.cfg;
  Layout& L = p.lay;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  // flags, inexact rows, of which overflowed, rows the merge spilled, items the sampled
  // selection handed to the exact one
  L.status = take(8 * sizeof(uint32_t));
  const size_t nb_stride = (size_t(1) << p.bucket_bits) + 1;
  if (p.use_tc) {
    // the orders, kept from rece_loss_fwd until rece_loss_bwd has run
    L.px = take(sizeof(int32_t) * c.n_r * c.N);
    L.py = take(sizeof(int32_t) * c.n_r * c.C);
  }
  // the sorted copies that the backward's band products read (the B operands) outlive
  // the forward
  if (p.tc_dy) L.xs = take(sizeof(uint16_t) * size_t(c.n_r) * c.N * c.d);
  if (p.tc_dx) {
    L.ys = take(sizeof(uint16_t) * size_t(tc_ys_rows(int64_t(c.n_r) * c.C)) * c.d);
    L.kept = take(sizeof(int2) * size_t(c.n_r) * c.N * c.k);
    L.kept_off = take(sizeof(int32_t) * size_t(c.n_r) * c.N * (size_t(p.kept_slices) + 1));
    L.pos_logit = take(sizeof(float) * size_t(c.N));
  }
  const size_t region = off;
  L.bx = take(sizeof(int32_t) * c.n_r * c.N);
  L.by = take(sizeof(int32_t) * c.n_r * c.C);
  if (!p.use_tc) {
    L.px = take(sizeof(int32_t) * c.n_r * c.N);
    L.py = take(sizeof(int32_t) * c.n_r * c.C);
  }
  L.bstart_x = take(sizeof(int32_t) * c.n_r * nb_stride);
  L.bstart_y = take(sizeof(int32_t) * c.n_r * nb_stride);
  // the forward sorts (X and Y of every round) run as one batch, a histogram each
  L.sort_scratch = take(size_t(c.n_r) * (sort_hist_bytes(c.N, p.bucket_bits) +
                                         sort_hist_bytes(c.C, p.bucket_bits)));
  if (p.use_tc) {
    const size_t Q = size_t(tc_list_capacity(c.k));
    if (!p.tc_dy) L.xs = take(sizeof(uint16_t) * size_t(c.n_r) * c.N * c.d);
    if (!p.tc_dx) L.ys = take(sizeof(uint16_t) * size_t(tc_ys_rows(int64_t(c.n_r) * c.C)) * c.d);
    L.inv_x = take(sizeof(int32_t) * c.n_r * c.N);
    L.chunk_y = take(sizeof(int32_t) * c.n_r * c.C);
    L.inv_y = take(sizeof(int32_t) * c.n_r * c.C);  // the merge's test for the positive
    L.tc_list = take(sizeof(int2) * size_t(c.n_r) * c.N * Q);
    L.tc_count = take(sizeof(int4) * c.n_r * c.N);
    L.tc_theta = take(sizeof(float) * c.n_r * c.N);
    if (p.tc_scores) L.scores = take(sizeof(float) * size_t(c.n_r) * c.N * p.score_width);
    L.spill_rows = take(sizeof(int32_t) * size_t(c.N));
    if (p.tc_sampled) L.redo_list = take(sizeof(int32_t) * size_t(tc_select_items(p)));
    L.spill_scratch = take(merge_tc_spill_bytes(c.n_r, c.k));
  } else {
    L.list_score = take(sizeof(float) * size_t(c.n_r) * c.N * c.k);
    L.list_item = take(sizeof(int32_t) * size_t(c.n_r) * c.N * c.k);
  }
  L.row_loss_tmp = take(sizeof(float) * c.N);
  L.fwd_end = off;
  off = region;
  layout_pairs(p, off);
  if (p.tc_dy) L.pos_parts = take(sizeof(float) * size_t(c.N) * c.d);
  if (p.dx_split > 0)
    L.dx_parts = take(sizeof(float) * size_t(c.n_r) * p.dx_split * size_t(c.N) * c.d);
  L.bwd_end = off;
  L.total = L.fwd_end > L.bwd_end ? L.fwd_end : L.bwd_end;
}

// The kernels read X, Y, B with 16-byte vector loads and write dX, dY with 16-byte stores
// and bulk copies: every matrix must start on a 16-byte boundary (NULL ones are skipped).
bool aligned16(std::initializer_list<const void*> ptrs) {
  for (const void* q : ptrs)
    if (q && (reinterpret_cast<uintptr_t>(q) & 15u) != 0) return false;
  return true;
}
constexpr const char* kMisaligned = "X, Y, B, dX and dY must be 16-byte aligned";

rece_status_t check_plan_ws(rece_plan_t plan, const void* ws, size_t ws_bytes) {
  if (!plan) return fail(RECE_ERR_INVALID_ARG, "plan is NULL");
  if (!ws) return fail(RECE_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(RECE_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (ws_bytes < plan->lay.total) return fail(RECE_ERR_WORKSPACE, "workspace too small");
  return RECE_OK;
}

// Plan of a sampled baseline (CE- / BCE+): the reduced loss's CUDA-core backward over
// k = n sampled slots.  Workspace: the status words, then the pair arrays (the forward's
// row-loss scratch shares their start: forward and backward are separate calls).
rece_status_t sampled_plan(int32_t kind, int64_t N, int64_t C, int32_t d, int32_t n,
                           int32_t mode, rece_plan_s& p) {
  if (kind != RECE_SAMPLED_CE_MINUS && kind != RECE_SAMPLED_BCE_PLUS)
    return fail(RECE_ERR_INVALID_ARG, "unknown sampled-loss kind");
  if (N < 0 || C < 1 || C >= kInt32Max || d < 1 || n < 0)
    return fail(RECE_ERR_INVALID_ARG, "bad sampled-loss sizes");
  if (mode != RECE_MODE_FP32_EXACT && mode != RECE_MODE_BF16)
    return fail(RECE_ERR_INVALID_ARG, "unknown mode");
  if (N * (int64_t(n) + 1) >= kInt32Max || N * int64_t(d) >= (int64_t(1) << 40))
    return fail(RECE_ERR_UNSUPPORTED, "sizes exceed 32-bit pair indexing");
  if (int64_t(d) + 2 * (int64_t(n) + 1) > 51200)
    return fail(RECE_ERR_UNSUPPORTED, "d + 2(n + 1) must be <= 51200");
  p = rece_plan_s();
  p.cfg.N = N;
  p.cfg.C = C;
  p.cfg.d = d;
  p.cfg.n_b = 1;
  p.cfg.n_c = 1;
  p.cfg.n_ec = 0;
  p.cfg.n_r = 1;
  p.cfg.k = n;
  p.cfg.mode = static_cast<rece_mode_t>(mode);
  set_pair_sort(p);
  p.sigmoid_g = kind == RECE_SAMPLED_BCE_PLUS;
  size_t off = 0;
  p.lay.status = off;
  off += align256(4 * sizeof(uint32_t));
  p.lay.row_loss_tmp = off;
  const size_t fwd_end = off + align256(sizeof(float) * size_t(N));
  layout_pairs(p, off);
  p.lay.bwd_end = off;
  p.lay.fwd_end = fwd_end;
  p.lay.total = fwd_end > off ? fwd_end : off;
  return RECE_OK;
}

// Forward of the all-negatives mode: chunk tables, the rounds' window sums on the tensor
// cores, their combination with l+, the mean.  `selected`, when given, is set to -1 (no
// subset is chosen); the logits are not produced.
rece_status_t all_neg_fwd(const rece_plan_s& p, const void* X, const void* Y,
                          const int32_t* targets, char* ws, float* loss, float* row_loss,
                          int32_t* selected, float* lse, cudaStream_t st) {
  const auto& c = p.cfg;
  const Layout& L = p.lay;
  auto I = [&](size_t o) { return reinterpret_cast<int32_t*>(ws + o); };
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  float* rl = row_loss ? row_loss : reinterpret_cast<float*>(ws + L.row_loss_tmp);
  float2* ms = reinterpret_cast<float2*>(ws + L.ms);
  float* ls = reinterpret_cast<float*>(ws + L.lse_sorted);
  const bool f32 = c.mode == RECE_MODE_FP32_EXACT;
  stage_mark(p, RECE_STAGE_SELECT, 0, st);
  RECE_CUDA(launch_window_meta(I(L.py), I(L.inv_y), c.C, c.n_c, c.n_r, I(L.itemc), nullptr,
                               nullptr, c.C, nullptr, st),
            "item chunk tables");
  RECE_CUDA(launch_window_meta(I(L.px), I(L.inv_x), c.N, c.n_c, c.n_r, I(L.rowc), targets,
                               I(L.inv_y), c.C, I(L.pz), st),
            "row chunk tables");
  if (p.window_tc)
    RECE_CUDA(launch_window_lse_tc(p, ws + L.xs, ws + L.ys, I(L.itemc), I(L.rowc), I(L.pz), ms,
                                   status, st),
              "window sums (tcgen05)");
  else if (f32)
    RECE_CUDA(launch_window_lse_fma(p, static_cast<const float*>(X),
                                    static_cast<const float*>(Y), I(L.px), I(L.py), targets,
                                    I(L.itemc), I(L.rowc), ms, st),
              "window sums (fmaf)");
  else
    RECE_CUDA(launch_window_lse_fma(p, static_cast<const __nv_bfloat16*>(X),
                                    static_cast<const __nv_bfloat16*>(Y), I(L.px), I(L.py),
                                    targets, I(L.itemc), I(L.rowc), ms, st),
              "window sums (fmaf)");
  stage_mark(p, RECE_STAGE_SELECT, 1, st);
  stage_mark(p, RECE_STAGE_MERGE_LOSS, 0, st);
  if (f32)
    RECE_CUDA(launch_window_combine(p, static_cast<const float*>(X),
                                    static_cast<const float*>(Y), targets, I(L.inv_x), ms, lse,
                                    rl, ls, status, st),
              "rounds' log-sum-exp");
  else
    RECE_CUDA(launch_window_combine(p, static_cast<const __nv_bfloat16*>(X),
                                    static_cast<const __nv_bfloat16*>(Y), targets, I(L.inv_x),
                                    ms, lse, rl, ls, status, st),
              "rounds' log-sum-exp");
  if (selected && c.N > 0)
    RECE_CUDA(cudaMemsetAsync(selected, 0xFF, sizeof(int32_t) * size_t(c.N) * c.k, st),
              "selected");
  stage_mark(p, RECE_STAGE_MERGE_LOSS, 1, st);
  stage_mark(p, RECE_STAGE_MEAN, 0, st);
  RECE_CUDA(launch_mean(rl, c.N, loss, st), "mean");
  stage_mark(p, RECE_STAGE_MEAN, 1, st);
  return RECE_OK;
}

// Backward of the all-negatives mode: the positives' terms (written), then the window
// terms of dX and of dY, added round by round.
template <typename T>
rece_status_t all_neg_bwd_t(const rece_plan_s& p, const T* X, const T* Y,
                            const int32_t* targets, const float* lse, const float* dloss,
                            char* ws, float* dX, float* dY, cudaStream_t st) {
  const Layout& L = p.lay;
  auto I = [&](size_t o) { return reinterpret_cast<const int32_t*>(ws + o); };
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  const float* ls = reinterpret_cast<const float*>(ws + L.lse_sorted);
  stage_mark(p, RECE_STAGE_BWD_ROWS, 0, st);
  RECE_CUDA(launch_backward(*p.pos_plan, X, Y, targets, nullptr, lse, nullptr, dloss, ws, dX,
                            dY, status, st),
            "positives' backward");
  if (p.window_tc)
    RECE_CUDA(launch_window_grad_tc(p, false, ws + L.xs, ws + L.ys, I(L.itemc), I(L.rowc),
                                    I(L.pz), ls, I(L.px), dloss, dX,
                                    reinterpret_cast<float*>(ws + L.dx_parts), status, st),
              "window dX (tcgen05)");
  else
    RECE_CUDA(launch_window_grad_fma(p, false, X, Y, I(L.px), I(L.py), targets, I(L.itemc),
                                     I(L.rowc), lse, dloss, dX, st),
              "window dX (fmaf)");
  stage_mark(p, RECE_STAGE_BWD_ROWS, 1, st);
  stage_mark(p, RECE_STAGE_BWD_SORT, 0, st);
  stage_mark(p, RECE_STAGE_BWD_SORT, 1, st);
  stage_mark(p, RECE_STAGE_BWD_ITEMS, 0, st);
  if (p.window_tc)
    RECE_CUDA(launch_window_grad_tc(p, true, ws + L.xs, ws + L.ys, I(L.itemc), I(L.rowc),
                                    I(L.pz), ls, I(L.py), dloss, dY, nullptr, status, st),
              "window dY (tcgen05)");
  else
    RECE_CUDA(launch_window_grad_fma(p, true, X, Y, I(L.px), I(L.py), targets, I(L.itemc),
                                     I(L.rowc), lse, dloss, dY, st),
              "window dY (fmaf)");
  stage_mark(p, RECE_STAGE_BWD_ITEMS, 1, st);
  return RECE_OK;
}

rece_status_t all_neg_bwd(const rece_plan_s& p, const void* X, const void* Y,
                          const int32_t* targets, const float* lse, const float* dloss,
                          char* ws, float* dX, float* dY, cudaStream_t st) {
  if (p.cfg.mode == RECE_MODE_FP32_EXACT)
    return all_neg_bwd_t(p, static_cast<const float*>(X), static_cast<const float*>(Y), targets,
                         lse, dloss, ws, dX, dY, st);
  return all_neg_bwd_t(p, static_cast<const __nv_bfloat16*>(X),
                       static_cast<const __nv_bfloat16*>(Y), targets, lse, dloss, ws, dX, dY, st);
}

// The exact full cross-entropy on the tcgen05 tensor cores, where their window kernels
// take the shape (bf16, d a multiple of 64 up to 256): the all-negatives mode with one
// bucket, one chunk and one round is the full cross-entropy -- every item is in every
// row's window, counted once, the positive entering once as l+ -- so the op runs that
// mode's kernels through an internal plan.  The workspace holds the plan's workspace,
// then the one (zero) random vector its bucketing reads.  Returns NULL elsewhere (the
// CUDA-core kernels of full_ce.cu run).
rece_plan_t full_ce_window_plan(int64_t N, int64_t C, int32_t d, int32_t mode) {
  if (mode != RECE_MODE_BF16 || N < 1 || C < 1 || d % 64 != 0 || d > 256) return nullptr;
  rece_config_t cfg{};
  cfg.N = N;
  cfg.C = C;
  cfg.d = d;
  cfg.n_b = 1;
  cfg.n_c = 1;
  cfg.n_ec = 0;
  cfg.n_r = 1;
  cfg.k = 1;
  cfg.mode = RECE_MODE_BF16;
  cfg.flags = RECE_FLAG_ALL_NEGATIVES;
  rece_plan_t p = nullptr;
  char saved[sizeof(g_last_error)];
  memcpy(saved, g_last_error, sizeof(saved));
  if (rece_plan_create(&cfg, &p) != RECE_OK) p = nullptr;
  memcpy(g_last_error, saved, sizeof(saved));  // a shape it does not take is no error
  if (p && !p->window_tc) {
    rece_plan_destroy(p);
    p = nullptr;
  }
  return p;
}

struct FullCeWindow {
  rece_plan_t plan = nullptr;
  ~FullCeWindow() { rece_plan_destroy(plan); }
};

}  // namespace

void rece::set_last_error(const char* msg) { fail(RECE_OK, msg); }

extern "C" {

const char* rece_status_string(rece_status_t s) {
  switch (s) {
    case RECE_OK: return "RECE_OK";
    case RECE_ERR_INVALID_ARG: return "RECE_ERR_INVALID_ARG";
    case RECE_ERR_UNSUPPORTED: return "RECE_ERR_UNSUPPORTED";
    case RECE_ERR_WORKSPACE: return "RECE_ERR_WORKSPACE";
    case RECE_ERR_CUDA: return "RECE_ERR_CUDA";
    case RECE_ERR_DEVICE_INPUT: return "RECE_ERR_DEVICE_INPUT";
    case RECE_ERR_TIMEOUT: return "RECE_ERR_TIMEOUT";
    case RECE_ERR_NO_DEVICE: return "RECE_ERR_NO_DEVICE";
  }
  return "RECE_ERR_UNKNOWN";
}

const char* rece_last_error_string(void) { return g_last_error; }

rece_status_t rece_plan_create(const rece_config_t* cfg, rece_plan_t* out) {
  if (!cfg || !out) return fail(RECE_ERR_INVALID_ARG, "cfg or plan pointer is NULL");
  *out = nullptr;
  rece_config_t c = *cfg;
  if (c.n_b == 0 || c.n_c == 0) {
    // n_b = n_c = 0: the bucket count the RECE paper calls optimal for peak memory,
    // n_b* = sqrt(4 alpha_bc (1 + 2 n_ec) min(C, N)), at alpha_bc = 1 (n_c = n_b, the
    // ratio its experiments found best), as rece_optimal_buckets rounds and clamps it
    if (c.n_b != 0 || c.n_c != 0)
      return fail(RECE_ERR_INVALID_ARG,
                  "n_b and n_c must both be 0 (the pages' n_b* at alpha_bc = 1) or both >= 1");
    if (c.N >= 0 && c.C >= 1 && c.n_ec >= 0) {
      int32_t nb = 1, nc = 1;
      if (c.N > 0 && rece_optimal_buckets(c.N, c.C, c.n_ec, 1.0, &nb, &nc) != RECE_OK)
        return RECE_ERR_INVALID_ARG;
      c.n_b = nb;
      c.n_c = nc;
    }
  }
  if (c.N < 0 || c.C < 1 || c.C >= kInt32Max) return fail(RECE_ERR_INVALID_ARG, "N or C out of range");
  if (c.d < 1) return fail(RECE_ERR_INVALID_ARG, "d must be >= 1");
  if (c.n_b < 1 || c.n_b > (1 << kMaxDigitBits))
    return fail(RECE_ERR_INVALID_ARG, "n_b must be in [1, 4096]");
  if (c.n_r < 1 || c.n_r > 8) return fail(RECE_ERR_INVALID_ARG, "n_r must be in [1, 8]");
  if (c.k < 1 || c.k > 4096) return fail(RECE_ERR_INVALID_ARG, "k must be in [1, 4096]");
  if (c.n_ec < 0) return fail(RECE_ERR_INVALID_ARG, "n_ec must be >= 0");
  if (c.n_c < 1 || c.n_c > c.C || (c.N > 0 && c.n_c > c.N))
    return fail(RECE_ERR_INVALID_ARG, "n_c must be in [1, min(N, C)]");
  if (c.mode != RECE_MODE_FP32_EXACT && c.mode != RECE_MODE_BF16)
    return fail(RECE_ERR_INVALID_ARG, "unknown mode");
  if ((c.flags & ~(RECE_FLAG_FMA_SCORES | RECE_FLAG_ALL_NEGATIVES)) != 0)
    return fail(RECE_ERR_INVALID_ARG, "unknown flag");
  if (c.N * (int64_t(c.k) + 1) >= kInt32Max || c.N * c.n_r >= kInt32Max ||
      c.C * c.n_r >= kInt32Max || c.N * c.d >= (int64_t(1) << 40))
    return fail(RECE_ERR_UNSUPPORTED, "sizes exceed 32-bit pair indexing");
  if (int64_t(c.n_r) * c.k > 8192) return fail(RECE_ERR_UNSUPPORTED, "n_r * k must be <= 8192");

  rece_plan_s* p = new (std::nothrow) rece_plan_s();
  if (!p) return fail(RECE_ERR_INVALID_ARG, "out of host memory");
  p->cfg = c;
  p->x_chunk_max = c.N > 0 ? ceil_div(c.N, c.n_c) : 0;
  p->y_chunk_max = ceil_div(c.C, c.n_c);
  p->w_max = 0;
  for (int64_t ch = 0; ch < c.n_c; ++ch) {
    const int64_t w = window_len(ch, c.C, c.n_c, c.n_ec);
    if (w > p->w_max) p->w_max = w;
  }
  p->sel_rows = 0;
  for (int G = 8; G >= 1; G >>= 1) {
    if (select_fma_smem_bytes(G, c.d, p->w_max) <= kMaxSmem) {
      p->sel_rows = G;
      break;
    }
  }
  if (p->sel_rows == 0 && !(c.flags & RECE_FLAG_ALL_NEGATIVES)) {
    delete p;
    return fail(RECE_ERR_UNSUPPORTED, "chunk window too long for the selection kernel");
  }
  p->bucket_bits = bits_for(c.n_b);
  set_pair_sort(*p);
  p->sigmoid_g = false;
  p->timed = false;
  for (void*& e : p->stage_events) e = nullptr;
  p->kept_slices = 0;
  for (int64_t ch = 0; ch < c.n_c; ++ch) {
    const int64_t w0 = chunk_start(ch - c.n_ec < 0 ? 0 : ch - c.n_ec, c.C, c.n_c);
    const int64_t w1 = chunk_start(ch + c.n_ec + 1 > c.n_c ? c.n_c : ch + c.n_ec + 1, c.C, c.n_c);
    const int64_t sl = w1 > w0 ? ((w1 - 1) >> 6) - (w0 >> 6) + 1 : 0;
    if (sl > p->kept_slices) p->kept_slices = int32_t(sl);
  }
  p->all_neg = (c.flags & RECE_FLAG_ALL_NEGATIVES) != 0;
  p->pos_plan = nullptr;
  // the tensor-core path groups each row's kept entries by slice of its window
  // (the selection's 16-bit histogram counts hold windows of fewer than 65536 items)
  p->use_tc = tc_supported(*p) &&
              (p->w_max < 65536 || (c.flags & RECE_FLAG_ALL_NEGATIVES) != 0);
  // dX on the tensor cores where gathering catalogue rows is the slow way: large d, or a
  // sorted catalogue that does not fit in half of L2; the merge groups each row's kept
  // entries by slice of its window for it
  // at large d the window scores are computed once and stored (a d-deep dot product per
  // score outweighs writing and reading it back)
  p->tc_scores = p->use_tc && c.d >= 1024;
  // the fused selection: a sampled threshold and one streaming pass where each pass's
  // multiply and stream cost outweigh emitting about twice k entries per row instead of
  // about k (measured: 4.2 -> 2.4 ms at the 4M-item workload, d = 256; no gain at d = 64
  // or 128, where the epilogue's per-score work, not the passes, bounds the kernel)
  p->tc_sampled = p->use_tc && !p->tc_scores && c.d >= 256;
  p->score_width = p->tc_scores ? scores_tc_width(*p) : 0;
  p->tc_dx = p->use_tc && p->kept_slices <= kMaxKeptSlices &&
             (c.d >= 256 || 2.0 * double(c.C) * c.d > 64.0 * 1024 * 1024);
  p->window_tc = false;
  if (p->all_neg) {
    // the window sums on tcgen05 where those kernels take the shape (bf16, d a multiple of
    // 64 up to 256), else on the CUDA cores (fmaf chains: fp32 mode, the FMA flag, wide d)
    p->window_tc = window_tc_supported(*p);
    p->tc_dx = false;
    p->tc_scores = false;
    p->tc_sampled = false;
    p->score_width = 0;
    // the positives' coefficients and their dY go through the pair backward (k = 0)
    rece_plan_s* q = new (std::nothrow) rece_plan_s();
    if (!q) {
      delete p;
      return fail(RECE_ERR_INVALID_ARG, "out of host memory");
    }
    *q = *p;
    q->cfg.k = 0;
    q->all_neg = false;
    q->use_tc = false;
    q->timed = false;
    q->pos_plan = nullptr;
    set_pair_sort(*q);
    p->pos_plan = q;
  } else if (p->use_tc && merge_tc_warp_bytes(c.n_r, c.k) > 200 * 1024) {
    delete p;
    return fail(RECE_ERR_UNSUPPORTED, "n_r * k too large for the tensor-core merge");
  }
  p->tc_dy = false;
  if (p->tc_dx && !p->all_neg && c.d >= 128) {
    // dY as band products too wherever dX is (from d = 128: each x row gathered per pair
    // is 2d bytes and the pairs need a sort by item, while the band's builders cost the
    // same per slab whatever d; measured 8.4 -> 4.8 ms at the 4M-item workload, d = 256);
    // the positives' dY through a pair backward of k = 0 that shares the pair region (N
    // pairs fit where N (k + 1) do)
    rece_plan_s* q = new (std::nothrow) rece_plan_s();
    if (!q) {
      delete p;
      return fail(RECE_ERR_INVALID_ARG, "out of host memory");
    }
    *q = *p;
    q->cfg.k = 0;
    q->use_tc = q->tc_dx = q->tc_dy = q->tc_scores = false;
    q->timed = false;
    q->pos_plan = nullptr;
    set_pair_sort(*q);
    p->pos_plan = q;
    p->tc_dy = true;
  }
  p->dx_split = p->tc_dx ? dx_tc_split(*p) : 0;
  build_layout(*p);
  if (p->tc_dy) {
    p->pos_plan->lay = p->lay;  // the main plan's pair arrays and status words
    p->pos_plan->carry_g = p->carry_g && p->pos_plan->carry_g;
  }
  *out = p;
  return RECE_OK;
}

void rece_plan_destroy(rece_plan_t plan) {
  if (plan) delete plan->pos_plan;
  delete plan;
}

rece_status_t rece_plan_set_stage_events(rece_plan_t plan, void* const* events) {
  if (!plan) return fail(RECE_ERR_INVALID_ARG, "plan is NULL");
  plan->timed = events != nullptr;
  for (int i = 0; i < 2 * RECE_NUM_STAGES; ++i) {
    plan->stage_events[i] = events ? events[i] : nullptr;
    if (events && !events[i]) {
      plan->timed = false;
      return fail(RECE_ERR_INVALID_ARG, "NULL event handle");
    }
  }
  return RECE_OK;
}

uint64_t rece_kernel_launch_count(void) { return g_launches.load(); }

rece_status_t rece_plan_get_config(rece_plan_t plan, rece_config_t* cfg) {
  if (!plan || !cfg) return fail(RECE_ERR_INVALID_ARG, "NULL argument");
  *cfg = plan->cfg;
  return RECE_OK;
}

rece_status_t rece_plan_workspace_size(rece_plan_t plan, size_t* bytes) {
  if (!plan || !bytes) return fail(RECE_ERR_INVALID_ARG, "NULL argument");
  *bytes = plan->lay.total;
  return RECE_OK;
}

rece_status_t rece_plan_workspace_layout(rece_plan_t plan, rece_workspace_layout_t* l) {
  if (!plan || !l) return fail(RECE_ERR_INVALID_ARG, "NULL argument");
  l->status = plan->lay.status;
  l->bucket_x = plan->lay.bx;
  l->bucket_y = plan->lay.by;
  l->perm_x = plan->lay.px;
  l->perm_y = plan->lay.py;
  l->bucket_start_y = plan->lay.bstart_y;
  l->bucket_start_stride = (size_t(1) << plan->bucket_bits) + 1;
  return RECE_OK;
}

rece_status_t rece_plan_paths(rece_plan_t plan, uint32_t* paths) {
  if (!plan || !paths) return fail(RECE_ERR_INVALID_ARG, "NULL argument");
  *paths = (plan->use_tc ? RECE_PATH_TENSOR_CORES : 0u) |
           (plan->tc_dx ? RECE_PATH_DX_TENSORS : 0u) |
           (plan->tc_scores ? RECE_PATH_STORED_SCORES : 0u) |
           (plan->all_neg ? RECE_PATH_ALL_NEGATIVES : 0u) |
           (plan->tc_dy ? RECE_PATH_DY_TENSORS : 0u) |
           (plan->dx_split > 0 ? RECE_PATH_DX_PARTS : 0u) |
           (plan->tc_sampled ? RECE_PATH_SAMPLED_SELECT : 0u) |
           (plan->all_neg && !plan->window_tc ? RECE_PATH_WINDOW_FMA : 0u);
  return RECE_OK;
}

rece_status_t rece_draw_projections(rece_plan_t plan, uint64_t seed, uint64_t step, void* B,
                                    void* stream) {
  if (!plan) return fail(RECE_ERR_INVALID_ARG, "NULL plan");
  if (!B) return fail(RECE_ERR_INVALID_ARG, "NULL B");
  const auto& c = plan->cfg;
  const int64_t count = int64_t(c.n_r) * c.n_b * c.d;
  RECE_CUDA(launch_draw_projections(seed, step, count, c.mode == RECE_MODE_BF16, B,
                                    static_cast<cudaStream_t>(stream)),
            "draw projections");
  return RECE_OK;
}

rece_status_t rece_bucketize_sort(rece_plan_t plan, const void* B, const void* X, const void* Y,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  rece_status_t s = check_plan_ws(plan, workspace, workspace_bytes);
  if (s != RECE_OK) return s;
  const auto& c = plan->cfg;
  if (!B || !Y || (c.N > 0 && !X)) return fail(RECE_ERR_INVALID_ARG, "NULL input");
  if (!aligned16({B, X, Y})) return fail(RECE_ERR_INVALID_ARG, kMisaligned);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const Layout& L = plan->lay;
  RECE_CUDA(cudaMemsetAsync(ws + L.status, 0, 8 * sizeof(uint32_t), st), "status reset");
  int32_t* bx = reinterpret_cast<int32_t*>(ws + L.bx);
  int32_t* by = reinterpret_cast<int32_t*>(ws + L.by);
  stage_mark(*plan, RECE_STAGE_BUCKETIZE, 0, st);
  if (c.mode == RECE_MODE_FP32_EXACT) {
    RECE_CUDA(launch_bucketize_fma(static_cast<const float*>(X), c.N, c.d,
                                   static_cast<const float*>(B), c.n_b, c.n_r, bx, st),
              "bucketize X");
    RECE_CUDA(launch_bucketize_fma(static_cast<const float*>(Y), c.C, c.d,
                                   static_cast<const float*>(B), c.n_b, c.n_r, by, st),
              "bucketize Y");
  } else if (plan->use_tc) {
    RECE_CUDA(launch_bucketize_tc(*plan, X, Y, B, bx, by,
                                  reinterpret_cast<uint32_t*>(ws + L.status), st),
              "bucketize (tcgen05)");
  } else {
    RECE_CUDA(launch_bucketize_fma(static_cast<const __nv_bfloat16*>(X), c.N, c.d,
                                   static_cast<const __nv_bfloat16*>(B), c.n_b, c.n_r, bx, st),
              "bucketize X");
    RECE_CUDA(launch_bucketize_fma(static_cast<const __nv_bfloat16*>(Y), c.C, c.d,
                                   static_cast<const __nv_bfloat16*>(B), c.n_b, c.n_r, by, st),
              "bucketize Y");
  }
  stage_mark(*plan, RECE_STAGE_BUCKETIZE, 1, st);
  stage_mark(*plan, RECE_STAGE_SORT, 0, st);
  const size_t stride = (size_t(1) << plan->bucket_bits) + 1;
  SortSeg segs[kMaxSortSegs];
  char* hist = ws + L.sort_scratch;
  for (int r = 0; r < c.n_r; ++r) {
    for (int side = 0; side < 2; ++side) {
      const int64_t M = side == 0 ? c.N : c.C;
      SortSeg& g = segs[2 * r + side];
      g = SortSeg{};
      g.keys = (side == 0 ? bx : by) + int64_t(r) * M;
      g.M = M;
      g.hist = reinterpret_cast<int32_t*>(hist);
      hist += sort_hist_bytes(M, plan->bucket_bits);
      g.start = reinterpret_cast<int32_t*>(ws + (side == 0 ? L.bstart_x : L.bstart_y)) + r * stride;
      g.out_ids = reinterpret_cast<int32_t*>(ws + (side == 0 ? L.px : L.py)) + int64_t(r) * M;
    }
  }
  RECE_CUDA(launch_sort_batch(segs, 2 * c.n_r, 0, plan->bucket_bits, false, st),
            "sort X and Y");
  if (plan->all_neg) {
    // sorted bf16 copies for the tcgen05 window kernels; the inverse orders either way
    RECE_CUDA(launch_permute_rows(X, c.N, plan->window_tc ? c.d : 0,
                                  reinterpret_cast<const int32_t*>(ws + L.px), c.n_r, c.n_c,
                                  plan->window_tc ? ws + L.xs : nullptr,
                                  reinterpret_cast<int32_t*>(ws + L.inv_x), nullptr, st),
              "permute X");
    RECE_CUDA(launch_permute_rows(Y, c.C, plan->window_tc ? c.d : 0,
                                  reinterpret_cast<const int32_t*>(ws + L.py), c.n_r, c.n_c,
                                  plan->window_tc ? ws + L.ys : nullptr,
                                  reinterpret_cast<int32_t*>(ws + L.inv_y), nullptr, st),
              "permute Y");
  } else if (plan->use_tc) {
    RECE_CUDA(launch_permute_rows(X, c.N, c.d, reinterpret_cast<const int32_t*>(ws + L.px),
                                  c.n_r, c.n_c, ws + L.xs,
                                  reinterpret_cast<int32_t*>(ws + L.inv_x), nullptr, st),
              "permute X");
    RECE_CUDA(launch_permute_rows(Y, c.C, c.d, reinterpret_cast<const int32_t*>(ws + L.py),
                                  c.n_r, c.n_c, ws + L.ys,
                                  reinterpret_cast<int32_t*>(ws + L.inv_y),
                                  reinterpret_cast<int32_t*>(ws + L.chunk_y), st),
              "permute Y");
    // the copy's padding to whole 128-row groups (read by the selection's tiles, masked)
    const int64_t rows = int64_t(c.n_r) * c.C, padded = tc_ys_rows(rows);
    if (padded > rows)
      RECE_CUDA(cudaMemsetAsync(ws + L.ys + size_t(rows) * c.d * 2, 0,
                                size_t(padded - rows) * c.d * 2, st),
                "pad Y copy");
  }
  stage_mark(*plan, RECE_STAGE_SORT, 1, st);
  return RECE_OK;
}

rece_status_t rece_loss_fwd(rece_plan_t plan, const void* X, const void* Y,
                            const int32_t* targets, void* workspace, size_t workspace_bytes,
                            float* loss, float* row_loss, int32_t* selected, float* lse,
                            float* logits, void* stream) {
  rece_status_t s = check_plan_ws(plan, workspace, workspace_bytes);
  if (s != RECE_OK) return s;
  const auto& c = plan->cfg;
  if (!loss || !Y || (c.N > 0 && (!X || !targets || (!selected && !plan->all_neg) || !lse)))
    return fail(RECE_ERR_INVALID_ARG, "NULL input or output");
  if (!aligned16({X, Y})) return fail(RECE_ERR_INVALID_ARG, kMisaligned);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const Layout& L = plan->lay;
  if (plan->all_neg) return all_neg_fwd(*plan, X, Y, targets, ws, loss, row_loss, selected, lse, st);
  const int32_t* px = reinterpret_cast<const int32_t*>(ws + L.px);
  const int32_t* py = reinterpret_cast<const int32_t*>(ws + L.py);
  float* ls = reinterpret_cast<float*>(ws + L.list_score);
  int32_t* li = reinterpret_cast<int32_t*>(ws + L.list_item);
  float* rl = row_loss ? row_loss : reinterpret_cast<float*>(ws + L.row_loss_tmp);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  if (c.mode == RECE_MODE_FP32_EXACT) {
    const float* Xf = static_cast<const float*>(X);
    const float* Yf = static_cast<const float*>(Y);
    stage_mark(*plan, RECE_STAGE_SELECT, 0, st);
    RECE_CUDA(launch_select_fma(*plan, Xf, Yf, targets, px, py, ls, li, st), "select");
    stage_mark(*plan, RECE_STAGE_SELECT, 1, st);
    stage_mark(*plan, RECE_STAGE_MERGE_LOSS, 0, st);
    RECE_CUDA(launch_merge_loss(*plan, Xf, Yf, targets, ls, li, selected, lse, rl, logits, status, st),
              "merge/loss");
  } else if (plan->use_tc) {
    const __nv_bfloat16* Xb = static_cast<const __nv_bfloat16*>(X);
    const __nv_bfloat16* Yb = static_cast<const __nv_bfloat16*>(Y);
    int2* list = reinterpret_cast<int2*>(ws + L.tc_list);
    int4* cnt = reinterpret_cast<int4*>(ws + L.tc_count);
    float* theta = reinterpret_cast<float*>(ws + L.tc_theta);
    stage_mark(*plan, RECE_STAGE_SELECT, 0, st);
    if (plan->tc_scores)
      RECE_CUDA(launch_scores_select_tc(*plan, ws + L.xs, ws + L.ys,
                                        reinterpret_cast<float*>(ws + L.scores), list, cnt, theta,
                                        status, st),
                "scores + select (tcgen05)");
    else
      RECE_CUDA(launch_select_tc(*plan, ws + L.xs, ws + L.ys, list, cnt, theta,
                                 reinterpret_cast<int32_t*>(ws + L.redo_list), status + 4,
                                 status, st),
                "select (tcgen05)");
    stage_mark(*plan, RECE_STAGE_SELECT, 1, st);
    stage_mark(*plan, RECE_STAGE_MERGE_LOSS, 0, st);
    RECE_CUDA(launch_merge_tc(*plan, Xb, Yb, targets, py,
                              reinterpret_cast<const int32_t*>(ws + L.inv_x),
                              reinterpret_cast<const int32_t*>(ws + L.inv_y),
                              reinterpret_cast<const int32_t*>(ws + L.chunk_y), list, cnt, theta,
                              selected,
                              plan->tc_dx ? reinterpret_cast<int2*>(ws + L.kept) : nullptr,
                              plan->tc_dx ? reinterpret_cast<int32_t*>(ws + L.kept_off) : nullptr,
                              plan->tc_dx ? reinterpret_cast<float*>(ws + L.pos_logit) : nullptr,
                              plan->kept_slices + 1, lse, rl, logits, status,
                              reinterpret_cast<int32_t*>(ws + L.spill_rows), ws + L.spill_scratch,
                              st),
              "merge/loss (tcgen05 lists)");
  } else {
    const __nv_bfloat16* Xb = static_cast<const __nv_bfloat16*>(X);
    const __nv_bfloat16* Yb = static_cast<const __nv_bfloat16*>(Y);
    stage_mark(*plan, RECE_STAGE_SELECT, 0, st);
    RECE_CUDA(launch_select_fma(*plan, Xb, Yb, targets, px, py, ls, li, st), "select");
    stage_mark(*plan, RECE_STAGE_SELECT, 1, st);
    stage_mark(*plan, RECE_STAGE_MERGE_LOSS, 0, st);
    RECE_CUDA(launch_merge_loss(*plan, Xb, Yb, targets, ls, li, selected, lse, rl, logits, status, st),
              "merge/loss");
  }
  stage_mark(*plan, RECE_STAGE_MERGE_LOSS, 1, st);
  stage_mark(*plan, RECE_STAGE_MEAN, 0, st);
  RECE_CUDA(launch_mean(rl, c.N, loss, st), "mean");
  stage_mark(*plan, RECE_STAGE_MEAN, 1, st);
  return RECE_OK;
}

rece_status_t rece_loss_bwd(rece_plan_t plan, const void* X, const void* Y,
                            const int32_t* targets, const int32_t* selected, const float* lse,
                            const float* logits, const float* dloss, void* workspace,
                            size_t workspace_bytes, float* dX, float* dY, void* stream) {
  rece_status_t s = check_plan_ws(plan, workspace, workspace_bytes);
  if (s != RECE_OK) return s;
  const auto& c = plan->cfg;
  if (!Y || !dY ||
      (c.N > 0 && (!X || !targets || (!selected && !plan->all_neg) || !lse || !dloss || !dX)))
    return fail(RECE_ERR_INVALID_ARG, "NULL input or output");
  if (!aligned16({X, Y, dX, dY})) return fail(RECE_ERR_INVALID_ARG, kMisaligned);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + plan->lay.status);
  if (plan->all_neg) return all_neg_bwd(*plan, X, Y, targets, lse, dloss, ws, dX, dY, st);
  if (c.mode == RECE_MODE_FP32_EXACT)
    RECE_CUDA(launch_backward(*plan, static_cast<const float*>(X), static_cast<const float*>(Y),
                              targets, selected, lse, logits, dloss, ws, dX, dY, status, st),
              "backward");
  else
    RECE_CUDA(launch_backward(*plan, static_cast<const __nv_bfloat16*>(X),
                              static_cast<const __nv_bfloat16*>(Y), targets, selected, lse,
                              logits, dloss, ws, dX, dY, status, st),
              "backward");
  return RECE_OK;
}

rece_status_t rece_full_ce_workspace_size(int64_t N, int64_t C, int32_t d, int32_t mode,
                                          size_t* bytes) {
  if (!bytes || N < 0 || C < 1 || d < 1 || (mode != RECE_MODE_FP32_EXACT && mode != RECE_MODE_BF16))
    return fail(RECE_ERR_INVALID_ARG, "bad full-CE arguments");
  FullCeWindow w;
  w.plan = full_ce_window_plan(N, C, d, mode);
  if (w.plan)
    *bytes = align256(w.plan->lay.total) + align256(sizeof(uint16_t) * size_t(d));
  else
    *bytes = align256(2 * sizeof(uint32_t)) + align256(sizeof(float) * size_t(N));
  return RECE_OK;
}

rece_status_t rece_full_ce_fwd(int64_t N, int64_t C, int32_t d, int32_t mode, const void* X,
                               const void* Y, const int32_t* targets, void* workspace,
                               size_t workspace_bytes, float* loss, float* row_loss, float* lse,
                               void* stream) {
  size_t need = 0;
  rece_status_t s = rece_full_ce_workspace_size(N, C, d, mode, &need);
  if (s != RECE_OK) return s;
  if (!workspace || workspace_bytes < need) return fail(RECE_ERR_WORKSPACE, "workspace too small");
  if (!loss || !Y || (N > 0 && (!X || !targets || !lse)))
    return fail(RECE_ERR_INVALID_ARG, "NULL input or output");
  if (!aligned16({X, Y})) return fail(RECE_ERR_INVALID_ARG, kMisaligned);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  FullCeWindow w;
  w.plan = full_ce_window_plan(N, C, d, mode);
  if (w.plan) {  // tcgen05: the all-negatives kernels at one bucket, chunk and round
    const size_t pb = align256(w.plan->lay.total);
    char* B = ws + pb;
    RECE_CUDA(cudaMemsetAsync(B, 0, sizeof(uint16_t) * size_t(d), st), "unit vector");
    rece_status_t r = rece_bucketize_sort(w.plan, B, X, Y, ws, pb, stream);
    if (r != RECE_OK) return r;
    return rece_loss_fwd(w.plan, X, Y, targets, ws, pb, loss, row_loss, nullptr, lse, nullptr,
                         stream);
  }
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  float* rl = row_loss ? row_loss : reinterpret_cast<float*>(ws + align256(2 * sizeof(uint32_t)));
  RECE_CUDA(cudaMemsetAsync(status, 0, 2 * sizeof(uint32_t), st), "status reset");
  if (mode == RECE_MODE_FP32_EXACT)
    RECE_CUDA(launch_full_ce_fwd(N, C, d, static_cast<const float*>(X),
                                 static_cast<const float*>(Y), targets, rl, lse, status, st),
              "full CE forward");
  else
    RECE_CUDA(launch_full_ce_fwd(N, C, d, static_cast<const __nv_bfloat16*>(X),
                                 static_cast<const __nv_bfloat16*>(Y), targets, rl, lse, status,
                                 st),
              "full CE forward");
  RECE_CUDA(launch_mean(rl, N, loss, st), "mean");
  return RECE_OK;
}

rece_status_t rece_full_ce_bwd(int64_t N, int64_t C, int32_t d, int32_t mode, const void* X,
                               const void* Y, const int32_t* targets, const float* lse,
                               const float* dloss, void* workspace, size_t workspace_bytes,
                               float* dX, float* dY, void* stream) {
  size_t need = 0;
  rece_status_t s = rece_full_ce_workspace_size(N, C, d, mode, &need);
  if (s != RECE_OK) return s;
  if (!workspace || workspace_bytes < need) return fail(RECE_ERR_WORKSPACE, "workspace too small");
  if (!Y || !dY || (N > 0 && (!X || !targets || !lse || !dloss || !dX)))
    return fail(RECE_ERR_INVALID_ARG, "NULL input or output");
  if (!aligned16({X, Y, dX, dY})) return fail(RECE_ERR_INVALID_ARG, kMisaligned);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  FullCeWindow w;
  w.plan = full_ce_window_plan(N, C, d, mode);
  if (w.plan)  // the forward left the sorted copies and tables in the workspace
    return rece_loss_bwd(w.plan, X, Y, targets, nullptr, lse, nullptr, dloss, workspace,
                         align256(w.plan->lay.total), dX, dY, stream);
  if (mode == RECE_MODE_FP32_EXACT)
    RECE_CUDA(launch_full_ce_bwd(N, C, d, static_cast<const float*>(X),
                                 static_cast<const float*>(Y), targets, lse, dloss, dX, dY, st),
              "full CE backward");
  else
    RECE_CUDA(launch_full_ce_bwd(N, C, d, static_cast<const __nv_bfloat16*>(X),
                                 static_cast<const __nv_bfloat16*>(Y), targets, lse, dloss, dX,
                                 dY, st),
              "full CE backward");
  return RECE_OK;
}

rece_status_t rece_optimal_buckets(int64_t N, int64_t C, int32_t n_ec, double alpha_bc,
                                   int32_t* n_b, int32_t* n_c) {
  if (!n_b || !n_c || N < 1 || C < 1 || n_ec < 0 || !(alpha_bc > 0.0))
    return fail(RECE_ERR_INVALID_ARG, "bad optimal-bucket arguments");
  const double mn = double(N < C ? N : C);
  double b = std::floor(std::sqrt(4.0 * alpha_bc * (1.0 + 2.0 * n_ec) * mn) + 0.5);
  b = b < 1.0 ? 1.0 : (b > double(1 << kMaxDigitBits) ? double(1 << kMaxDigitBits) : b);
  double c = std::floor(b / alpha_bc + 0.5);
  c = c < 1.0 ? 1.0 : (c > mn ? mn : c);
  *n_b = int32_t(b);
  *n_c = int32_t(c);
  return RECE_OK;
}

rece_status_t rece_memory_model_elements(int64_t N, int64_t C, int32_t n_ec, int32_t n_r,
                                         double alpha_bc, double* elements) {
  if (!elements || N < 1 || C < 1 || n_ec < 0 || n_r < 1 || !(alpha_bc > 0.0))
    return fail(RECE_ERR_INVALID_ARG, "bad memory-model arguments");
  const double mn = double(N < C ? N : C), mx = double(N < C ? C : N);
  *elements = 2.0 * n_r * std::sqrt(alpha_bc * (1.0 + 2.0 * n_ec) * mn) * mx;
  return RECE_OK;
}

rece_status_t rece_sampled_workspace_size(int32_t kind, int64_t N, int64_t C, int32_t d,
                                          int32_t n, int32_t mode, size_t* bytes) {
  if (!bytes) return fail(RECE_ERR_INVALID_ARG, "bytes is NULL");
  rece_plan_s p;
  rece_status_t s = sampled_plan(kind, N, C, d, n, mode, p);
  if (s != RECE_OK) return s;
  *bytes = p.lay.total;
  return RECE_OK;
}

rece_status_t rece_sampled_fwd(int32_t kind, int64_t N, int64_t C, int32_t d, int32_t n,
                               int32_t mode, const void* X, const void* Y,
                               const int32_t* targets, const int32_t* negatives,
                               void* workspace, size_t workspace_bytes, float* loss,
                               float* row_loss, float* logits, float* lse, void* stream) {
  rece_plan_s p;
  rece_status_t s = sampled_plan(kind, N, C, d, n, mode, p);
  if (s != RECE_OK) return s;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < p.lay.total)
    return fail(RECE_ERR_WORKSPACE, "workspace NULL, unaligned or too small");
  if (!loss || !Y || (N > 0 && (!X || !targets || (n > 0 && !negatives) ||
                                (kind == RECE_SAMPLED_CE_MINUS && !lse))))
    return fail(RECE_ERR_INVALID_ARG, "NULL input or output");
  if (!aligned16({X, Y})) return fail(RECE_ERR_INVALID_ARG, kMisaligned);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + p.lay.status);
  float* rl = row_loss ? row_loss : reinterpret_cast<float*>(ws + p.lay.row_loss_tmp);
  RECE_CUDA(cudaMemsetAsync(status, 0, 4 * sizeof(uint32_t), st), "status reset");
  if (mode == RECE_MODE_FP32_EXACT)
    RECE_CUDA(launch_sampled_fwd(kind, N, C, d, n, static_cast<const float*>(X),
                                 static_cast<const float*>(Y), targets, negatives, logits, lse,
                                 rl, status, st),
              "sampled forward");
  else
    RECE_CUDA(launch_sampled_fwd(kind, N, C, d, n, static_cast<const __nv_bfloat16*>(X),
                                 static_cast<const __nv_bfloat16*>(Y), targets, negatives,
                                 logits, lse, rl, status, st),
              "sampled forward");
  RECE_CUDA(launch_mean(rl, N, loss, st), "mean");
  return RECE_OK;
}

rece_status_t rece_sampled_bwd(int32_t kind, int64_t N, int64_t C, int32_t d, int32_t n,
                               int32_t mode, const void* X, const void* Y,
                               const int32_t* targets, const int32_t* negatives,
                               const float* logits, const float* lse, const float* dloss,
                               void* workspace, size_t workspace_bytes, float* dX, float* dY,
                               void* stream) {
  rece_plan_s p;
  rece_status_t s = sampled_plan(kind, N, C, d, n, mode, p);
  if (s != RECE_OK) return s;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < p.lay.total)
    return fail(RECE_ERR_WORKSPACE, "workspace NULL, unaligned or too small");
  if (!Y || !dY || (N > 0 && (!X || !targets || (n > 0 && !negatives) || !dloss || !dX ||
                              (kind == RECE_SAMPLED_CE_MINUS && !lse))))
    return fail(RECE_ERR_INVALID_ARG, "NULL input or output");
  if (!aligned16({X, Y, dX, dY})) return fail(RECE_ERR_INVALID_ARG, kMisaligned);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + p.lay.status);
  if (mode == RECE_MODE_FP32_EXACT)
    RECE_CUDA(launch_backward(p, static_cast<const float*>(X), static_cast<const float*>(Y),
                              targets, negatives, lse, logits, dloss, ws, dX, dY, status, st),
              "sampled backward");
  else
    RECE_CUDA(launch_backward(p, static_cast<const __nv_bfloat16*>(X),
                              static_cast<const __nv_bfloat16*>(Y), targets, negatives, lse,
                              logits, dloss, ws, dX, dY, status, st),
              "sampled backward");
  return RECE_OK;
}

rece_status_t rece_get_device_status(const void* workspace, uint32_t* device_flags,
                                     void* stream) {
  if (!workspace || !device_flags) return fail(RECE_ERR_INVALID_ARG, "NULL argument");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RECE_CUDA(cudaStreamSynchronize(st), "stream synchronize");
  RECE_CUDA(cudaMemcpy(device_flags, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost),
            "status read");
  if (*device_flags & RECE_DEVICE_TIMEOUT) return fail(RECE_ERR_TIMEOUT, "device wait timed out");
  if (*device_flags & RECE_DEVICE_BAD_TARGET) return fail(RECE_ERR_DEVICE_INPUT, "device input error");
  return RECE_OK;
}

}  // extern "C"
