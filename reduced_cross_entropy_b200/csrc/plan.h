// plan.h -- host-side plan of the RECE library and the internal kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "rece.h"

namespace rece {

// Counting-sort geometry: one CTA sorts a tile of kSortTile elements (8 warps x 256).
constexpr int kSortTile = 2048;
constexpr int kSortThreads = 256;
constexpr int kMaxDigitBits = 12;  // up to 4096 buckets in one pass

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int bits_for(int64_t n_values) {  // digit bits so that values 0..n_values-1 fit
  int b = 0;
  while ((int64_t(1) << b) < n_values) ++b;
  return b;
}

// Scratch of one counting sort pass over M elements with `bits`-bit digits.
inline size_t sort_scratch_bytes(int64_t M, int bits) {
  int64_t tiles = ceil_div(M > 0 ? M : 1, kSortTile);
  int64_t digits = int64_t(1) << bits;
  return align256(sizeof(int32_t) * size_t(digits * tiles)) +
         align256(sizeof(int32_t) * size_t(digits + 1));
}

// One independent counting sort of a batch (see launch_sort_batch): its keys (read by id,
// or in position order), M elements, histogram scratch (digits x tiles ints), the
// digits + 1 starts it writes, and its outputs.  `tiles` is filled in by the launcher.
struct SortSeg {
  const int32_t* keys;
  const int32_t* in_ids;
  int64_t M;
  int32_t* hist;
  int64_t tiles;
  int32_t* start;
  int32_t* out_ids;
  int32_t* out_keys;
  const float* payload;
  float* out_payload;
};
constexpr int kMaxSortSegs = 16;
struct SortBatch {
  SortSeg seg[kMaxSortSegs];
  int n, shift, bits;
  bool in_order;
};
// Histogram scratch of one batch segment of M elements.
inline size_t sort_hist_bytes(int64_t M, int bits) {
  return align256(sizeof(int32_t) * size_t(ceil_div(M, kSortTile) << bits));
}

// dY by gathered rows: an item whose run holds more pairs than this is summed by a whole
// CTA (its run split among the warps, the parts added in warp order) instead of one warp.
constexpr int kLongRunPairs = 256;

struct Layout {
  size_t status = 0;
  // forward region (from rece_bucketize_sort to the end of rece_loss_fwd)
  size_t bx = 0, by = 0, px = 0, py = 0, bstart_y = 0, bstart_x = 0;
  size_t sort_scratch = 0;
  size_t list_score = 0, list_item = 0, row_loss_tmp = 0;
  // tensor-core path (bf16 mode): sorted row copies, inverse orders, candidate lists
  size_t xs = 0, ys = 0, inv_x = 0, chunk_y = 0, tc_list = 0, tc_count = 0, tc_theta = 0,
         spill_rows = 0, spill_scratch = 0, scores = 0,
         redo_list = 0;  // work items the sampled selection hands to the exact one
  size_t fwd_end = 0;
  // backward region (rece_loss_bwd), overlaps the forward region
  size_t e_key = 0, e_g = 0, e_perm_a = 0, e_perm_b = 0, e_sorted_key = 0, e_key_b = 0,
         e_sorted_g = 0, e_g_b = 0, e_item_start = 0, e_scratch = 0,
         e_long = 0;  // dY: count and list of the items with runs of > kLongRunPairs pairs
  size_t bwd_end = 0;
  // tensor-core dX (and dY): kept from rece_loss_fwd to rece_loss_bwd (not aliased): the
  // sorted copies of Y (and X) -- xs, ys above, placed here then -- the kept entries by
  // (round, sorted row) with their slice starts, and each row's positive logit
  size_t kept = 0, kept_off = 0, pos_logit = 0;
  // all-negatives mode, kept from rece_loss_fwd to rece_loss_bwd: the chunk tables, the
  // positives' sorted positions, lse per round in sorted order; forward only: the rounds'
  // (max, sum) pairs and the inverse orders of Y
  size_t itemc = 0, rowc = 0, pz = 0, lse_sorted = 0, ms = 0, inv_y = 0,
         dx_parts = 0;  // (also the tensor-core dX's parts when split, backward region)
  // tensor-core dY: the positives' per-segment partial sums [N][d] (backward region)
  size_t pos_parts = 0;
  size_t total = 0;
};

}  // namespace rece

struct rece_plan_s {
  rece_config_t cfg;
  int64_t x_chunk_max;  // ceil(N / n_c)
  int64_t y_chunk_max;  // ceil(C / n_c)
  int64_t w_max;        // longest window (items)
  int32_t sel_rows;     // rows per CTA of the exact selection kernel
  int32_t bucket_bits;  // digit bits of the bucket sort
  int32_t item_bits;    // key bits of the backward item sort (values 0..C)
  int32_t item_passes;  // LSD passes of that sort (digits of at most 12 bits)
  int32_t item_pass_bits;  // digit bits of every pass but the last
  int64_t entries;      // N * (k + 1): (row, item) pairs of the backward
  bool carry_g;         // the pair sort carries g (its array would not stay in L2)
  bool sigmoid_g;       // backward coefficients sigmoid(l) - [positive] (BCE+), else softmax
  bool use_tc;          // bf16 mode on the tcgen05 kernels
  bool tc_dx;           // ... and dX of the backward on them too
  bool tc_dy;           // ... and dY (band products; positives through pos_plan's pairs)
  int dx_split;         // tensor-core dX: 0 one launch per round, S > 0 K splits into parts
  bool tc_scores;       // ... with the window scores computed once and stored (large d)
  bool tc_sampled;      // ... else the fused selection's threshold from a 1/8 sample of
                        // the window (one streaming pass; d >= 256), or exact (three)
  int64_t score_width;  // columns of the stored scores per row (longest union, padded)
  int32_t kept_slices;  // most 64-position slices one window touches
  bool all_neg;         // RECE_FLAG_ALL_NEGATIVES: Algorithm 1 as printed, no top-k
  bool window_tc;       // ... its window sums and gradients on tcgen05 (else CUDA cores)
  rece_plan_s* pos_plan;  // all-negatives mode and tensor-core dY: the positives' pair
                          // backward (k = 0)
  rece::Layout lay;
  void* stage_events[2 * RECE_NUM_STAGES];  // optional timing hook (cudaEvent_t)
  bool timed;
};

namespace rece {

// Process-wide count of kernel launches (statistics only).
void count_launches(int n);

// Records the stage's start (end = 0) or end (end = 1) event when timing is on.
inline void stage_mark(const rece_plan_s& p, int stage, int end, cudaStream_t st) {
  if (p.timed) cudaEventRecord(static_cast<cudaEvent_t>(p.stage_events[2 * stage + end]), st);
}

// ---------------------------------------------------------------- launchers
// All launchers enqueue on `st` and return the launch error (cudaSuccess if none).

// The random vectors B [n_r][n_b][d] (count elements) of call `step` of a run seeded with
// `seed`: SplitMix64 outputs, Box-Muller normals (projections.cu), fp32 or bf16.
cudaError_t launch_draw_projections(uint64_t seed, uint64_t step, int64_t count, bool bf16,
                                    void* B, cudaStream_t st);

// K1: bucket[r][i] = argmax_b <B[r][b], V[i]> (fmaf chain, ties to lowest b).
template <typename T>
cudaError_t launch_bucketize_fma(const T* V, int64_t M, int d, const T* B, int n_b, int n_r,
                                 int32_t* bucket, cudaStream_t st);

// K2: one stable counting-sort pass over M elements.  Element p carries id
// (in_ids ? in_ids[p] : p) and key keys[id]; it is ordered by digit (key >> shift) &
// ((1 << bits) - 1).  Writes out_ids (the new order of ids), optionally the sorted keys
// (out_keys[p] = keys[out_ids[p]]), a carried payload (out_payload[p] =
// payload[out_ids[p]]) and digit_start[0..2^bits] (first output position of every digit;
// digit_start[2^bits] = M).
// With in_order, element p's key and payload are keys[p] and payload[p] (a previous pass
// wrote them in the order of its output) instead of being looked up by id.
cudaError_t sort_pairs_by_item(const rece_plan_s& p, int64_t E, const int32_t* key,
                               const float* g, int32_t* perm_a, int32_t* perm_b, int32_t* key_b,
                               float* g_b, int32_t* sorted_key, float* sorted_g, void* scratch,
                               const int32_t** sorted_id, cudaStream_t st);
cudaError_t launch_sort_batch(const SortSeg* segs, int n, int shift, int bits, bool in_order,
                              cudaStream_t st);
cudaError_t launch_sort_pass(const int32_t* keys, const int32_t* in_ids, int64_t M, int shift,
                             int bits, void* scratch, int32_t* out_ids, int32_t* out_keys,
                             int32_t* digit_start, cudaStream_t st,
                             const float* payload = nullptr, float* out_payload = nullptr,
                             bool in_order = false);

// start[j] = first position of a key >= j in the sorted keys, for j = 0..n_vals (so the
// keys equal to j occupy [start[j], start[j+1])).
cudaError_t launch_segment_starts(const int32_t* sorted, int64_t M, int32_t n_vals,
                                  int32_t* start, cudaStream_t st);

// K3 (fmaf-chain CUDA-core version): per-round top-k lists of every row.
template <typename T>
cudaError_t launch_select_fma(const rece_plan_s& p, const T* X, const T* Y,
                              const int32_t* targets, const int32_t* px, const int32_t* py,
                              float* list_score, int32_t* list_item, cudaStream_t st);

// K4: merge the rounds' lists, de-duplicate, keep k, loss per row.
template <typename T>
cudaError_t launch_merge_loss(const rece_plan_s& p, const T* X, const T* Y,
                              const int32_t* targets, const float* list_score,
                              const int32_t* list_item, int32_t* selected, float* lse,
                              float* row_loss, float* logits, uint32_t* status,
                              cudaStream_t st);

// K7: loss[0] = sum(row_loss) / N in a fixed order.
cudaError_t launch_mean(const float* row_loss, int64_t N, float* loss, cudaStream_t st);

// K5: backward.
template <typename T>
cudaError_t launch_backward(const rece_plan_s& p, const T* X, const T* Y,
                            const int32_t* targets, const int32_t* selected, const float* lse,
                            const float* logits, const float* dloss, char* ws, float* dX,
                            float* dY, uint32_t* status, cudaStream_t st);

// Sampled baselines (sampled.cu): logits [N][n+1], lse (CE-) and row losses.
size_t sampled_fwd_warp_bytes(int d, int n);
template <typename T>
cudaError_t launch_sampled_fwd(int kind, int64_t N, int64_t C, int d, int n, const T* X,
                               const T* Y, const int32_t* targets, const int32_t* neg,
                               float* logits, float* lse, float* row_loss, uint32_t* status,
                               cudaStream_t st);

// K6: exact full cross-entropy.
template <typename T>
cudaError_t launch_full_ce_fwd(int64_t N, int64_t C, int d, const T* X, const T* Y,
                               const int32_t* targets, float* row_loss, float* lse,
                               uint32_t* status, cudaStream_t st);
template <typename T>
cudaError_t launch_full_ce_bwd(int64_t N, int64_t C, int d, const T* X, const T* Y,
                               const int32_t* targets, const float* lse, const float* dloss,
                               float* dX, float* dY, cudaStream_t st);

}  // namespace rece
