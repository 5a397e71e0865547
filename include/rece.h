/*
 * rece.h -- C ABI of the B200 (sm_100a) reduced cross-entropy library.
 *
 * The loss is RECE ("RECE: Reduced Cross-Entropy Loss for Large-Catalogue Sequential
 * Recommenders", section 3, Algorithm 1) with the top-k subset of SCE ("Scalable
 * Cross-Entropy Loss for Sequential Recommendations with Large Item Catalogs",
 * abstract):
 *
 *   1. project the model outputs X [N x d] and the catalogue Y [C x d] onto n_b random
 *      vectors and give every row the bucket with the largest inner product;
 *   2. sort the rows of X and of Y by bucket (stable);
 *   3. split both sorted arrays into n_c equal chunks and score every row of chunk c
 *      against the items of chunks c-n_ec .. c+n_ec, over n_r independent rounds;
 *   4. keep, per row, the k highest-scoring negatives (the positive excluded, rounds
 *      united and de-duplicated, ties to the lower item id);
 *   5. softmax cross-entropy over the positive plus those negatives, mean over rows;
 *   6. gradients dX and dY of that loss (selection held constant).
 * The N x C logit matrix is never formed.  An exact fused full cross-entropy
 * (equations 3 and 4 of the RECE paper) is provided for comparison.
 *
 * Conventions shared by every call
 *   - Pointers marked "device" point to GPU memory the caller owns; the library never
 *     allocates device memory.  Matrices are row-major and contiguous, and X, Y, B, dX
 *     and dY start on a 16-byte boundary (RECE_ERR_INVALID_ARG otherwise).
 *   - Element type of X, Y, B: fp32 in RECE_MODE_FP32_EXACT, bf16 in RECE_MODE_BF16.
 *     Losses, log-sum-exps and gradients are always fp32.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Calls
 *     only enqueue work; nothing synchronises except rece_get_device_status.
 *   - Host-side argument errors are returned at once and enqueue nothing.  Bad device
 *     data (a target outside [0, C)) cannot be seen on the host: the kernels record it
 *     in the workspace's status word, the affected rows get a NaN loss, and
 *     rece_get_device_status reports it.
 *   - No global state: plans are independent host objects; one plan may be used from
 *     one thread at a time.
 */
#ifndef RECE_H_
#define RECE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RECE_API __attribute__((visibility("default")))
#else
#define RECE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RECE_OK = 0,
  RECE_ERR_INVALID_ARG = 1,  /* a size, pointer or config field is out of range */
  RECE_ERR_UNSUPPORTED = 2,  /* valid, but not implemented for this mode/shape */
  RECE_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
  RECE_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, copy, ...) */
  RECE_ERR_DEVICE_INPUT = 5, /* device-side input error recorded (see status word) */
  RECE_ERR_TIMEOUT = 6,      /* a bounded device wait gave up */
  RECE_ERR_NO_DEVICE = 7     /* no usable sm_100 device for this call */
} rece_status_t;

typedef enum {
  /* fp32 inputs; every score that decides an index (bucket, selection) is the fixed-
   * order chain s = fmaf(a[t], b[t], s), t = 0..d-1 from s = 0, so indices are
   * reproducible bit for bit by any implementation of the same chain. */
  RECE_MODE_FP32_EXACT = 0,
  /* bf16 inputs; scores come from the tcgen05 tensor cores (fp32 accumulation). */
  RECE_MODE_BF16 = 1
} rece_mode_t;

/* rece_config_t.flags */
#define RECE_FLAG_FMA_SCORES 0x1u /* bf16 mode: use the fmaf-chain CUDA-core kernels for
                                     the scores as well (bit-exact on bf16 inputs) */
/* Algorithm 1 as printed [RECE section 3]: every item of a row's chunk windows is a
 * negative (no top-k; k is not used), and a pair computed in cnt of the n_r rounds
 * enters each round's sum as exp(l - ln cnt) [the rounds paragraph], the positive left
 * out of the window sums (it enters once, as l+):
 *   lse_i = log(exp(l+) + sum_r sum_{j in W_r(i), j != z_i} exp(l_ij) / cnt_ij).
 * The window sums are never stored; the backward recomputes them: on the tcgen05 tensor
 * cores in bf16 mode with d a multiple of 64 up to 256, else (fp32 mode, bf16 with
 * RECE_FLAG_FMA_SCORES, other widths) on the CUDA cores with the fixed-order fmaf chain of
 * the scores (RECE_PATH_WINDOW_FMA).  rece_loss_fwd writes no logits and fills `selected`
 * (which may be NULL) with -1; rece_loss_bwd ignores `selected` and `logits` (either may be
 * NULL). */
#define RECE_FLAG_ALL_NEGATIVES 0x2u

/* Bits of the device status word (rece_get_device_status). */
#define RECE_DEVICE_BAD_TARGET 0x1u /* some target outside [0, C) */
#define RECE_DEVICE_TIMEOUT 0x2u    /* a bounded wait inside a kernel gave up */
#define RECE_DEVICE_INEXACT 0x4u    /* bf16 tensor-core mode: some rows' top-k could not be
                                       certified exact (a candidate list overflowed or a
                                       threshold was above the k-th kept score); the 32-bit
                                       word after the status word counts those rows, the
                                       next one those whose candidate list overflowed */

typedef struct {
  int64_t N;     /* rows (batch x sequence), >= 0 */
  int64_t C;     /* catalogue size, >= 1 */
  int32_t d;     /* embedding width, >= 1 (bf16 mode: multiple of 16 for tcgen05) */
  int32_t n_b;   /* random vectors per round, 1 .. 4096; 0 together with n_c = 0: the
                    pages' n_b* at alpha_bc = 1 (see rece_plan_create) */
  int32_t n_c;   /* chunks, 1 .. min(N, C) (any n_c <= C when N = 0); 0 with n_b = 0 */
  int32_t n_ec;  /* neighbouring chunks on each side, >= 0 */
  int32_t n_r;   /* rounds, 1 .. 8 */
  int32_t k;     /* negatives kept per row, 1 .. 4096 */
  int32_t mode;  /* rece_mode_t */
  uint32_t flags;
} rece_config_t;

typedef struct rece_plan_s* rece_plan_t;

/* Byte offsets of the intermediate arrays inside the workspace (valid between
 * rece_bucketize_sort and the next rece_loss_bwd on that workspace).  The status word
 * is always at offset 0. */
typedef struct {
  size_t status;   /* uint32 device status word */
  size_t bucket_x; /* int32 [n_r][N]: bucket id of every row of X, per round */
  size_t bucket_y; /* int32 [n_r][C] */
  size_t perm_x;   /* int32 [n_r][N]: row ids in stable bucket order, per round */
  size_t perm_y;   /* int32 [n_r][C] */
  size_t bucket_start_y; /* int32 [n_r][bucket_start_stride]: first sorted position of
                            each bucket id b (entries b >= n_b hold C) */
  size_t bucket_start_stride; /* elements per round: 2^ceil(log2 n_b) + 1 */
} rece_workspace_layout_t;

/* Validate cfg and build a host-side plan (no CUDA call, no device memory).
 * cfg, plan: host pointers.  On success *plan owns a host object freed by
 * rece_plan_destroy.  RECE_ERR_INVALID_ARG / RECE_ERR_UNSUPPORTED on a bad config.
 * n_b = n_c = 0 asks for the bucket count the RECE paper calls optimal for peak memory
 * [RECE section 3, the paragraph before Algorithm 1]: n_b* at alpha_bc = n_b / n_c = 1
 * (section 5: n_c = n_b gave the best quality for a memory budget), i.e. n_b = n_c =
 * rece_optimal_buckets(N, C, n_ec, 1.0) (1 when N = 0); only one of them 0 is
 * RECE_ERR_INVALID_ARG.  rece_plan_get_config returns the values chosen. */
RECE_API rece_status_t rece_plan_create(const rece_config_t* cfg, rece_plan_t* plan);
RECE_API void rece_plan_destroy(rece_plan_t plan);

/* The plan's configuration as resolved by rece_plan_create (n_b and n_c filled in when
 * they were 0).  cfg: host pointer.  RECE_ERR_INVALID_ARG for a NULL argument. */
RECE_API rece_status_t rece_plan_get_config(rece_plan_t plan, rece_config_t* cfg);

/* Device workspace bytes the plan needs (one buffer, caller-allocated, 256-byte
 * aligned).  The same buffer serves rece_bucketize_sort, rece_loss_fwd and
 * rece_loss_bwd; rece_loss_bwd reuses the space the forward intermediates held. */
RECE_API rece_status_t rece_plan_workspace_size(rece_plan_t plan, size_t* bytes);
RECE_API rece_status_t rece_plan_workspace_layout(rece_plan_t plan, rece_workspace_layout_t* layout);

/* Which kernels a plan runs (host-side; no device work).  *paths receives the OR of:
 *   RECE_PATH_TENSOR_CORES  bf16 mode on tcgen05: bucketing and the window scores with
 *                           their selection (else the fmaf kernels);
 *   RECE_PATH_DX_TENSORS    dX of the backward as tcgen05 band products (large d or a
 *                           catalogue beyond half of L2; else gathered rows);
 *   RECE_PATH_STORED_SCORES window scores computed once and stored, then selected row by
 *                           row (d >= 1024; else recomputed in the fused selection);
 *   RECE_PATH_ALL_NEGATIVES the all-negatives mode (RECE_FLAG_ALL_NEGATIVES);
 *   RECE_PATH_DY_TENSORS    dY as tcgen05 band products as well (with RECE_PATH_DX_TENSORS;
 *                           else a stable pair sort and gathered rows);
 *   RECE_PATH_DX_PARTS      (with RECE_PATH_DX_TENSORS) the dX band products of all rounds
 *                           in one launch, each row tile's window split in parts that are
 *                           stored and then summed in a fixed order (when per-round
 *                           launches would leave their last wave part-empty);
 *   RECE_PATH_SAMPLED_SELECT the fused selection sets each row's threshold from a 1/8
 *                           sample of its window and streams the window once (d >= 256);
 *                           rows it cannot certify are selected again by the exact
 *                           three-pass kernel, so the result is the same either way;
 *   RECE_PATH_WINDOW_FMA    (with RECE_PATH_ALL_NEGATIVES) the window sums and their
 *                           gradients on the CUDA cores, with the fixed-order fmaf chain
 *                           of RECE_MODE_FP32_EXACT (fp32 mode, RECE_FLAG_FMA_SCORES, or a
 *                           width the tcgen05 window kernels do not take).
 * RECE_ERR_INVALID_ARG for a NULL argument. */
#define RECE_PATH_TENSOR_CORES 0x1u
#define RECE_PATH_DX_TENSORS 0x2u
#define RECE_PATH_STORED_SCORES 0x4u
#define RECE_PATH_ALL_NEGATIVES 0x8u  /* RECE_FLAG_ALL_NEGATIVES: window sums on tcgen05 */
#define RECE_PATH_DY_TENSORS 0x10u
#define RECE_PATH_DX_PARTS 0x20u
#define RECE_PATH_SAMPLED_SELECT 0x40u
#define RECE_PATH_WINDOW_FMA 0x80u  /* with RECE_PATH_ALL_NEGATIVES: window sums on the CUDA
                                       cores (fmaf chains), not tcgen05 */
RECE_API rece_status_t rece_plan_paths(rece_plan_t plan, uint32_t* paths);

/* Algorithm 1's randn step [RECE section 3, Algorithm 1: the random vectors], drawn on
 * the device: B [n_r][n_b][d] (device, in the plan's element type: fp32, or bf16 rounded
 * to nearest even from the fp32 value; caller-owned, any alignment rece_bucketize_sort
 * accepts) is filled with standard normals of call `step` of a run seeded with `seed`.
 * The stream is counter-based, so any element can be drawn alone and a call repeats
 * exactly: SplitMix64 [Steele, Lea, Flood, OOPSLA 2014] started at
 * s = mix(mix(seed) ^ step), whose i-th output is mix(s + (i+1) * 0x9E3779B97F4A7C15)
 * with mix(z) = z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27;
 * z *= 0x94D049BB133111EB; z ^= z >> 31; outputs x -> uniforms ((x >> 11) + 1) 2^-53 in
 * (0, 1]; element pair q by Box-Muller from outputs 2q and 2q+1: rho = sqrt(-2 ln u1),
 * theta = 6.283185307179586 u2, elements rho cos(theta), rho sin(theta) (fp64, then fp32),
 * in B's row-major order.  Enqueued on `stream`; B may be passed to rece_bucketize_sort
 * on the same stream right after.  Errors: NULL plan or B (RECE_ERR_INVALID_ARG), a
 * launch failure (RECE_ERR_CUDA). */
RECE_API rece_status_t rece_draw_projections(rece_plan_t plan, uint64_t seed, uint64_t step,
                                             void* B, void* stream);

/* Steps 1-2 [RECE section 3, Algorithm 1: random vectors, argmax bucketing, argsort].
 *   B  device, [n_r][n_b][d] random vectors (one set per round, N(0,1), afresh for every
 *      call as the paper does: rece_draw_projections draws them, or the caller does)
 *   X  device, [N][d];  Y device, [C][d]
 * Writes bucket ids and stable per-round orders into the workspace, and clears the
 * status word.  Must precede rece_loss_fwd on the same workspace and stream. */
RECE_API rece_status_t rece_bucketize_sort(rece_plan_t plan, const void* B, const void* X,
                                  const void* Y, void* workspace, size_t workspace_bytes,
                                  void* stream);

/* Steps 3-5 [RECE Algorithm 1: chunks, windows, logits, loss; SCE abstract: top-k].
 *   targets  device int32 [N], positive item of every row, in [0, C)
 *   loss     device fp32 [1]: mean over rows of the per-row loss (0 when N = 0)
 *   row_loss device fp32 [N] or NULL
 *   selected device int32 [N][k]: the kept negatives, -1 where a row has fewer than k
 *            candidates; in RECE_MODE_FP32_EXACT (and with RECE_FLAG_FMA_SCORES) best first
 *            (score descending, item id ascending), on the tensor-core path in a fixed
 *            order (by round, then by sorted catalogue position within each selection
 *            warpgroup's share) -- the set is the same, the order is deterministic
 *   lse      device fp32 [N]: log(exp(l+) + sum over selected exp(l)) per row
 *   logits   device fp32 [N][k+1] or NULL: the logits the loss used, the positive's
 *            first, then those of `selected` (-inf where selected is -1)
 * selected and lse (and logits, which spare the backward recomputing them) are what
 * rece_loss_bwd needs. */
RECE_API rece_status_t rece_loss_fwd(rece_plan_t plan, const void* X, const void* Y,
                            const int32_t* targets, void* workspace, size_t workspace_bytes,
                            float* loss, float* row_loss, int32_t* selected, float* lse,
                            float* logits, void* stream);

/* Step 6 [RECE equation (4) on the positive and the kept negatives]:
 *   g_ij = (exp(l_ij - lse_i) - [j == z_i]) * dloss / N
 *   logits device fp32 [N][k+1] from rece_loss_fwd, or NULL to recompute the l_ij
 *   dX_i = sum_j g_ij y_j,   dY_j = sum_i g_ij x_i
 *   dloss  device fp32 [1]: gradient of the caller's objective w.r.t. the mean loss
 *   dX     device fp32 [N][d], dY device fp32 [C][d]: overwritten (items no row touched
 *          get exactly 0).  Deterministic: no floating-point atomics. */
RECE_API rece_status_t rece_loss_bwd(rece_plan_t plan, const void* X, const void* Y,
                            const int32_t* targets, const int32_t* selected,
                            const float* lse, const float* logits, const float* dloss,
                            void* workspace, size_t workspace_bytes, float* dX, float* dY,
                            void* stream);

/* Exact full cross-entropy [RECE equations (3) and (4)], fused: the logits are formed
 * tile by tile on chip and never stored.  Arguments as above; mode picks the input
 * element type.  In bf16 mode with d a multiple of 64 up to 256 the op runs on the tcgen05
 * tensor cores as the all-negatives mode (RECE_FLAG_ALL_NEGATIVES) at n_b = n_c = n_r = 1
 * -- every item in every row's window, counted once, which is equation (3) -- and its
 * workspace then holds that mode's sorted copies and tables: rece_full_ce_bwd must get the
 * workspace rece_full_ce_fwd used, unchanged in between.  Elsewhere (fp32 mode, other
 * widths) it runs on the CUDA cores and the workspace holds the status word and the row
 * losses.  rece_full_ce_workspace_size gives the bytes for the shape and mode. */
RECE_API rece_status_t rece_full_ce_workspace_size(int64_t N, int64_t C, int32_t d, int32_t mode,
                                          size_t* bytes);
RECE_API rece_status_t rece_full_ce_fwd(int64_t N, int64_t C, int32_t d, int32_t mode, const void* X,
                               const void* Y, const int32_t* targets, void* workspace,
                               size_t workspace_bytes, float* loss, float* row_loss,
                               float* lse, void* stream);
RECE_API rece_status_t rece_full_ce_bwd(int64_t N, int64_t C, int32_t d, int32_t mode, const void* X,
                               const void* Y, const int32_t* targets, const float* lse,
                               const float* dloss, void* workspace, size_t workspace_bytes,
                               float* dX, float* dY, void* stream);

/* Bucket count for the least memory [RECE section 3, the paragraph before Algorithm 1]:
 *   n_b* = sqrt(4 alpha_bc (1 + 2 n_ec) min(C, N)),   alpha_bc = n_b / n_c,
 * rounded to the nearest integer and clamped to [1, 4096]; n_c* = n_b* / alpha_bc rounded,
 * clamped to [1, min(N, C)].  N is the row count (the pages' s * l).  Host only. */
RECE_API rece_status_t rece_optimal_buckets(int64_t N, int64_t C, int32_t n_ec, double alpha_bc,
                                            int32_t* n_b, int32_t* n_c);
/* The pages' memory model of the method at n_b* [same paragraph], in logit elements:
 *   2 r sqrt(alpha_bc (1 + 2 n_ec) min(C, N)) max(C, N),
 * against N * C for the full cross-entropy (ratio sqrt(min) / (2 r sqrt(alpha_bc (1 + 2 n_ec)))).
 * A model of Algorithm 1, which stores every chunk's logits; this library keeps them on
 * chip, so its workspace sits below the model.  Host only. */
RECE_API rece_status_t rece_memory_model_elements(int64_t N, int64_t C, int32_t n_ec, int32_t n_r,
                                                  double alpha_bc, double* elements);

/* Sampled baselines [RECE section 2, Related Work, equations (1) and (2)]: the loss of
 * row i over its positive z_i and n given negatives, with l = <x_i, y_j>:
 *   RECE_SAMPLED_CE_MINUS (eq. 2): loss_i = log(exp(l+) + sum_j exp(l_ij)) - l+
 *   RECE_SAMPLED_BCE_PLUS (eq. 1): loss_i = -log sigmoid(l+) - sum_j log(1 - sigmoid(l_ij))
 * L = (1/N) sum_i loss_i.  The caller draws the negatives (uniformly, in the pages'
 * setting); the library takes them as given:
 *   negatives  device int32 [N][n] (NULL when n = 0): ids in [0, C) or < 0 for padding
 *              (no term).  A sample equal to the row's positive is a negative like any
 *              other, and a repeated sample counts once per occurrence, as the sums are
 *              written.  Ids >= C and targets outside [0, C) set RECE_DEVICE_BAD_TARGET.
 *   mode       element type of X and Y (fp32 or bf16), arithmetic in fp32
 * Workspace (rece_sampled_workspace_size bytes, 256-byte aligned): the status word, then
 * the backward's pair arrays.  fwd writes loss [1], row_loss [N] (or NULL), logits
 * [N][n+1] (slot 0 the positive, slot s the negative s-1; padding 0; or NULL) and, for
 * CE-, lse [N] (required; unused and may be NULL for BCE+).  bwd takes fwd's logits (or
 * NULL: they are recomputed) and lse, and overwrites dX [N][d] and dY [C][d]:
 *   g_i+ = (p_i+ - 1) dloss/N,  g_ij = p_ij dloss/N,  p = exp(l - lse) (CE-), sigmoid(l) (BCE+)
 *   dX_i = g_i+ y_{z_i} + sum_j g_ij y_j,  dY_j = sum of g x_i over the pairs naming j,
 * deterministic (no floating-point atomics).  Limits: N (n+1) < 2^31, d + 2(n+1) <= 51200.
 * Host errors (bad sizes, kind or mode, NULL pointers, small workspace) return before
 * anything is launched. */
#define RECE_SAMPLED_CE_MINUS 0
#define RECE_SAMPLED_BCE_PLUS 1
RECE_API rece_status_t rece_sampled_workspace_size(int32_t kind, int64_t N, int64_t C, int32_t d,
                                                   int32_t n, int32_t mode, size_t* bytes);
RECE_API rece_status_t rece_sampled_fwd(int32_t kind, int64_t N, int64_t C, int32_t d, int32_t n,
                                        int32_t mode, const void* X, const void* Y,
                                        const int32_t* targets, const int32_t* negatives,
                                        void* workspace, size_t workspace_bytes, float* loss,
                                        float* row_loss, float* logits, float* lse,
                                        void* stream);
RECE_API rece_status_t rece_sampled_bwd(int32_t kind, int64_t N, int64_t C, int32_t d, int32_t n,
                                        int32_t mode, const void* X, const void* Y,
                                        const int32_t* targets, const int32_t* negatives,
                                        const float* logits, const float* lse,
                                        const float* dloss, void* workspace,
                                        size_t workspace_bytes, float* dX, float* dY,
                                        void* stream);

/* Stable bucket sort that allocates nothing (the pages have no counterpart: this is an
 * interface for callers, not a step of the method).  It is step 2's sort on its own, for
 * callers that cannot give the library device memory: code running inside another
 * application's fixed device-memory arena (a plugin or custom operator that is not
 * allowed to allocate), or a loop that cannot take an allocation's latency and implicit
 * synchronisation.  Its scratch (per-tile histograms) is a 4 MiB array of device memory
 * inside the library image; every GPU the library is used on holds it until the process
 * exits.
 *   bucket_ids   device int32 [M], values in [0, n_b); any other value, negative ones
 *                included, is sorted by its low ceil(log2 n_b) bits (two's complement),
 *                i.e. as the key (value & (2^ceil(log2 n_b) - 1)), stably
 *   order        device int32 [M]: element indices by (bucket asc, index asc)
 *   bucket_start device int32 [2^ceil(log2 n_b) + 1] or NULL: first position of every
 *                bucket id (entries from n_b on hold M)
 * Returns RECE_ERR_UNSUPPORTED, having launched nothing, when the per-2048-element-tile
 * histograms of M elements by 2^ceil(log2 n_b) buckets do not fit the 4 MiB (about
 * M * 2^ceil(log2 n_b) <= 2^31: M <= 520,192 at n_b = 4096, M <= 8,384,512 at n_b = 256).
 * The first call on a device looks up the array's device address (make that first call
 * before any stream capture) and keeps it for the rest of the process: after
 * cudaDeviceReset (or anything else that tears the device's primary context down) the kept
 * address is stale, so do not call this function again in that process.  All calls share
 * the array: calls whose GPU work can overlap (unordered streams or threads) race; order
 * them. */
RECE_API rece_status_t rece_bucket_sort_static(const int32_t* bucket_ids, int64_t M,
                                               int32_t n_b, int32_t* order,
                                               int32_t* bucket_start, void* stream);

/* Synchronises `stream`, then copies the workspace's status word to *device_flags
 * (RECE_DEVICE_* bits).  Returns RECE_ERR_TIMEOUT / RECE_ERR_DEVICE_INPUT when the
 * timeout / bad-target bit is set (RECE_DEVICE_INEXACT alone is informational and returns
 * RECE_OK), RECE_ERR_CUDA when the stream reports an error. */
RECE_API rece_status_t rece_get_device_status(const void* workspace, uint32_t* device_flags,
                                     void* stream);

/* Stages of the path that rece_plan_set_stage_events can time. */
#define RECE_STAGE_BUCKETIZE 0  /* step 1: projection + argmax, X and Y, all rounds */
#define RECE_STAGE_SORT 1       /* step 2: stable bucket sorts, all rounds */
#define RECE_STAGE_SELECT 2     /* steps 3-4: chunk scores + per-round top-k */
#define RECE_STAGE_MERGE_LOSS 3 /* steps 4-5: round merge, de-duplication, row losses */
#define RECE_STAGE_MEAN 4       /* step 5: mean over rows */
#define RECE_STAGE_BWD_ROWS 5   /* step 6: coefficients and dX, one row at a time */
#define RECE_STAGE_BWD_SORT 6   /* step 6: (item, row) pairs put in item order */
#define RECE_STAGE_BWD_ITEMS 7  /* step 6: dY, one item at a time */
#define RECE_NUM_STAGES 8

/* Optional timing hook: events points to 2 * RECE_NUM_STAGES cudaEvent_t handles (as
 * void*) owned by the caller; each later call records events[2s] on its stream just
 * before stage s and events[2s+1] just after it.  NULL switches the hook off.  The
 * handles must outlive their use; the plan does not own them. */
RECE_API rece_status_t rece_plan_set_stage_events(rece_plan_t plan, void* const* events);

/* Number of CUDA kernels this library has launched in the process so far (all plans,
 * all threads); lets a caller count the kernels in a timed region. */
RECE_API uint64_t rece_kernel_launch_count(void);

/* Static, human-readable name of a status code. */
RECE_API const char* rece_status_string(rece_status_t status);

/* Detail of the last error returned on the calling thread (a CUDA error name and the
 * failing step, or the argument that was rejected).  Thread-local, never NULL. */
RECE_API const char* rece_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* RECE_H_ */
