// tc.h -- internal interface of the tcgen05 (tensor-core) kernels of the bf16 mode.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "plan.h"

namespace rece {

// Tensor map of a row-major bf16 matrix [rows x cols] (cols a multiple of 64), boxes of
// 64 columns x box_rows rows, 128-byte swizzle (the K-major layout the MMA reads).
cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows);
// rows x cols bf16 matrices, `planes` of them one after another (cols a multiple of 64);
// box {64, box_rows, 1}, 128-byte swizzle; rows past the end read as zeros.
cudaError_t make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t cols,
                              uint64_t rows, uint64_t planes, uint32_t box_rows);
// A row-major bf16 matrix of groups x group_rows rows (cols a multiple of 64) seen as
// [groups][group_rows][cols]: one box is the first box_rows rows of box_groups consecutive
// groups, which lands in shared memory as box_rows * box_groups rows of a 128-byte-swizzled
// K-major tile; groups past the end read as zeros.
cudaError_t make_tmap_bf16_groups(CUtensorMap* map, const void* base, uint64_t cols,
                                  uint64_t groups, uint32_t group_rows, uint32_t box_rows,
                                  uint32_t box_groups);
int sm_count();
// out[i] += parts[0][i] + parts[1][i] + ... (n floats each, n % 4 == 0), in that order.
cudaError_t launch_add_parts(const float* parts, int64_t n, int nparts, float* out,
                             cudaStream_t st);


// bf16 mode without RECE_FLAG_FMA_SCORES and d a multiple of 64: the tcgen05 kernels run.
bool tc_supported(const rece_plan_s& p);

// K1 on tensor cores: bucket[r][i] = argmax_b <B[r][b], V[i]> for V = X and V = Y.
cudaError_t launch_bucketize_tc(const rece_plan_s& p, const void* X, const void* Y,
                                const void* B, int32_t* bx, int32_t* by, uint32_t* status,
                                cudaStream_t st);

// Sorted row copies (bf16) and inverse orders / per-round chunk of every row.
cudaError_t launch_permute_rows(const void* V, int64_t M, int d, const int32_t* perm, int n_r,
                                int n_c, void* Vs, int32_t* inv, int32_t* chunk,
                                cudaStream_t st);

// K3 on tensor cores: per (round, sorted row) the candidate list (score bits, sorted
// catalogue position), its count and threshold.
// The sorted copy Ys that the selection reads is padded to whole 128-row groups
// (tc_ys_rows of the n_r * C rows; the padding is zeroed by rece_bucketize_sort).  With
// p.tc_sampled a sampled pass sets each row's threshold and one pass emits; the items it
// could not certify (redo_list, *redo_count, at most tc_select_items) are done again by
// the exact kernel, which otherwise runs alone over every item.
int tc_list_capacity(int k);      // entries per (round, row): 4 sub-lists
int tc_sublist_capacity(int k);   // entries per sub-list
int64_t tc_ys_rows(int64_t rows);
int64_t tc_select_items(const rece_plan_s& p);
cudaError_t launch_select_tc(const rece_plan_s& p, const void* Xs, const void* Ys, int2* list,
                             int4* list_count, float* list_theta, int32_t* redo_list,
                             uint32_t* redo_count, uint32_t* status, cudaStream_t st);

// Steps 3-4 for large d (see scores_tc.cu): window scores once into S [n_r][N][width],
// then the exact per-row selection into the same lists as launch_select_tc.
int64_t scores_tc_width(const rece_plan_s& p);
cudaError_t launch_scores_select_tc(const rece_plan_s& p, const void* Xs, const void* Ys,
                                    float* S, int2* list, int4* list_count, float* list_theta,
                                    uint32_t* status, cudaStream_t st);

// K4 for the tensor-core lists: merge, select, loss, exactness check.  The kept entries
// go out by round and 64-position slice of the round's sorted catalogue: items
// (selected [N][k]) and logits ([N][k+1], or NULL), and for the backward, indexed by
// (round r, sorted row p): kept [n_r][N][k] = (sorted position, softmax probability as
// bf16 hi | lo << 16), kept_off [n_r][N][Sp] = slice starts of the row's window (entry S
// = the count); and pos_logit [N], each row's positive logit.
// Rows with more candidates than the fast path's shared buffer go through a spill list
// (spill_rows [N]) to a second launch with global scratch (merge_tc_spill_bytes).
size_t merge_tc_warp_bytes(int n_r, int k);
size_t merge_tc_spill_bytes(int n_r, int k);
constexpr int kMaxKeptSlices = 512;  // slices of one window the merge can group by
template <typename T>
cudaError_t launch_merge_tc(const rece_plan_s& p, const T* X, const T* Y, const int32_t* targets,
                            const int32_t* py, const int32_t* invX, const int32_t* invY,
                            const int32_t* chunkY, const int2* list, const int4* list_count,
                            const float* list_theta, int32_t* selected, int2* kept,
                            int32_t* kept_off, float* pos_logit, int Sp, float* lse,
                            float* row_loss, float* logits, uint32_t* status, int32_t* spill_rows,
                            void* spill_scratch, cudaStream_t st);

// dX of step 6 on tensor cores (see bwd_tc.cu): the positives' terms written, the
// rounds' added.  Needs the grouped merge outputs (kept, kept_off, pos_logit) and the
// sorted copy Ys.
template <typename T>
cudaError_t launch_dx_tc(const rece_plan_s& p, const T* Y, const int32_t* targets,
                         const float* lse, const float* dloss, char* ws, float* dX,
                         uint32_t* status, cudaStream_t st);

// 0: dX band products one launch per round, each adding into dX; S >= 1: one launch over
// (round, K split) into n_r S parts of dX (Layout::dx_parts), summed in order after.
int dx_tc_split(const rece_plan_s& p);

// dY of step 6 on tensor cores: the rounds' window terms, written by round 0 and added by
// the others (the positives' terms are added after).  Needs the grouped kept entries and
// the sorted copy Xs.
cudaError_t launch_dy_tc(const rece_plan_s& p, const float* dloss, char* ws, float* dY,
                         uint32_t* status, cudaStream_t st);

// All-negatives mode (Algorithm 1 as printed; window.cu, window_tc.cu).  Per-round chunk
// tables chunks[(r * n_r + s) * M + p] of the row (item) at sorted position p of round r,
// and for the rows the sorted position of their positive (pz [n_r][N], -1 for none).
cudaError_t launch_window_meta(const int32_t* perm, const int32_t* inv, int64_t M, int n_c,
                               int n_r, int32_t* chunks, const int32_t* targets,
                               const int32_t* invY, int64_t C, int32_t* pz, cudaStream_t st);
// bf16, d a multiple of 64 up to 256, at most 8 rounds.
bool window_tc_supported(const rece_plan_s& p);
// ms [n_r][N]: per round and sorted row, (max, sum) of exp(s)/cnt over its window terms.
cudaError_t launch_window_lse_tc(const rece_plan_s& p, const void* Xs, const void* Ys,
                                 const int32_t* itemc, const int32_t* rowc, const int32_t* pz,
                                 float2* ms, uint32_t* status, cudaStream_t st);
// lse and row losses from l+ and the rounds' (max, sum); lse also per round, sorted.
template <typename T>
cudaError_t launch_window_combine(const rece_plan_s& p, const T* X, const T* Y,
                                  const int32_t* targets, const int32_t* invX, const float2* ms,
                                  float* lse, float* row_loss, float* lse_sorted,
                                  uint32_t* status, cudaStream_t st);
// The all-negatives mode on the CUDA cores (window_fma.cu: fp32 mode, RECE_FLAG_FMA_SCORES,
// or bf16 widths the tcgen05 window kernels do not take), reading X and Y in place through
// the orders px, py: ms [n_r][N] as launch_window_lse_tc writes it, and the window terms
// of dX (dy = false) or dY (dy = true) added into `out` one round after another.
template <typename T>
cudaError_t launch_window_lse_fma(const rece_plan_s& p, const T* X, const T* Y,
                                  const int32_t* px, const int32_t* py, const int32_t* targets,
                                  const int32_t* itemc, const int32_t* rowc, float2* ms,
                                  cudaStream_t st);
template <typename T>
cudaError_t launch_window_grad_fma(const rece_plan_s& p, bool dy, const T* X, const T* Y,
                                   const int32_t* px, const int32_t* py, const int32_t* targets,
                                   const int32_t* itemc, const int32_t* rowc, const float* lse,
                                   const float* dloss, float* out, cudaStream_t st);
// The window terms of dX (dy = false, perm = px) or dY (dy = true, perm = py), added
// into `out` round by round (dX with `scratch` [n_r][N][d]: all rounds in one grid, then
// added in round order).
cudaError_t launch_window_grad_tc(const rece_plan_s& p, bool dy, const void* Xs,
                                  const void* Ys, const int32_t* itemc, const int32_t* rowc, const int32_t* pz,
                                  const float* lse_sorted, const int32_t* perm,
                                  const float* dloss, float* out, float* scratch,
                                  uint32_t* status, cudaStream_t st);

}  // namespace rece
