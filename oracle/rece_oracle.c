/*
 * rece_oracle.c -- plain, slow, CPU reference of the reduced cross-entropy loss.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA path is checked
 * against.  Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load it.  It shares no code, header, table or constant with the CUDA library, and
 * the CUDA library never calls it.
 *
 * Sources (cited by page title and section):
 *   [RECE]  "RECE: Reduced Cross-Entropy Loss for Large-Catalogue Sequential
 *           Recommenders", section 3 (Reduced Cross-Entropy): equations (3) and (4),
 *           Algorithm 1, and the paragraph before Algorithm 1 (rounds, duplicate pairs,
 *           neighbouring chunks).
 *           Section 2 (Related Work): equations (1) BCE+ and (2) CE-, the sampled
 *           baselines.
 *   [SCE]   "Scalable Cross-Entropy Loss for Sequential Recommendations with Large
 *           Item Catalogs", abstract (softmax approximated over a subset found by
 *           maximum inner product search, i.e. the top-k negatives per row).
 *
 * Precision.  Every decision that yields an integer (bucket argmax, candidate order)
 * is taken on fp32 scores, each formed by one fixed-order fused multiply-add chain
 *     s = 0; for t = 0..d-1: s = fmaf(a[t], b[t], s)
 * (both sides use this order so the indices they produce can be compared bit for
 * bit).  Loss values and gradients are computed in fp64 from the fp32 inputs.
 * Build with -ffp-contract=off and without fast-math.
 *
 * Readings of the pages (where they are silent or ambiguous):
 *   - chunk c of an M-element sorted array starts at ceil(c*M/n_c);
 *   - the window of chunk c is the union of chunks max(0,c-n_ec)..min(n_c-1,c+n_ec)
 *     of the sorted catalogue (edge chunks see fewer items);
 *   - the row's own positive item is never a negative;
 *   - candidates from all rounds are united and de-duplicated by item id (subtracting
 *     ln(count) from a logit seen count times, as the pages do, is the same thing);
 *   - the negatives kept are the k best candidates by (score descending, item id
 *     ascending); with fewer than k candidates all are kept;
 *   - selection and buckets are constants for the gradient;
 *   - the loss is the mean over rows; an empty batch has loss 0.
 *
 * Parity of every function here is pinned by tests that do not call this file's
 * arithmetic (brute force on exactly representable inputs, library sorts and argmax,
 * the full-CE identity, finite differences, invariants).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* One fp32 score: the fixed-order fmaf chain over the d coordinates. */
static float dot_f32(const float* a, const float* b, int32_t d) {
  float s = 0.0f;
  for (int32_t t = 0; t < d; ++t) s = fmaf(a[t], b[t], s);
  return s;
}

/* The same inner product in fp64 (for loss values and gradients). */
static double dot_f64(const float* a, const float* b, int32_t d) {
  double s = 0.0;
  for (int32_t t = 0; t < d; ++t) s += (double)a[t] * (double)b[t];
  return s;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* [RECE] Algorithm 1, the two argmax steps: bucket of row v = index of the random
 * vector b_k with the largest inner product <b_k, v>.  Ties go to the lowest k. */
void oracle_bucketize(const float* V, int64_t M, int32_t d, const float* B, int32_t n_b,
                      int32_t* bucket) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < M; ++i) {
    const float* v = V + i * (int64_t)d;
    int32_t best = 0;
    float best_s = dot_f32(B, v, d);
    for (int32_t b = 1; b < n_b; ++b) {
      float s = dot_f32(B + (int64_t)b * d, v, d);
      if (s > best_s) {
        best_s = s;
        best = b;
      }
    }
    bucket[i] = best;
  }
}

typedef struct {
  int32_t key;
  int32_t idx;
} key_idx_t;

static int cmp_key_idx(const void* pa, const void* pb) {
  const key_idx_t* a = (const key_idx_t*)pa;
  const key_idx_t* b = (const key_idx_t*)pb;
  if (a->key != b->key) return a->key < b->key ? -1 : 1;
  return a->idx < b->idx ? -1 : (a->idx > b->idx ? 1 : 0);
}

/* [RECE] Algorithm 1, the two argsort steps, read as a stable sort: perm lists the
 * element indices in order of (key ascending, original index ascending). */
void oracle_stable_argsort(const int32_t* keys, int64_t M, int32_t* perm) {
  key_idx_t* a = (key_idx_t*)malloc(sizeof(key_idx_t) * (size_t)(M > 0 ? M : 1));
  for (int64_t i = 0; i < M; ++i) {
    a[i].key = keys[i];
    a[i].idx = (int32_t)i;
  }
  qsort(a, (size_t)M, sizeof(key_idx_t), cmp_key_idx);
  for (int64_t i = 0; i < M; ++i) perm[i] = a[i].idx;
  free(a);
}

/* [RECE] Algorithm 1, chunk sets: element i of an M-long sorted array is in chunk c
 * when c*M/n_c <= i < (c+1)*M/n_c, so chunk c starts at ceil(c*M/n_c). */
int64_t oracle_chunk_start(int64_t c, int64_t M, int64_t n_c) {
  return (c * M + n_c - 1) / n_c;
}

typedef struct {
  float score;
  int32_t item;
} cand_t;

/* Candidate order of [SCE]: higher score first; equal scores by lower item id. */
static int cmp_cand(const void* pa, const void* pb) {
  const cand_t* a = (const cand_t*)pa;
  const cand_t* b = (const cand_t*)pb;
  if (a->score > b->score) return -1;
  if (a->score < b->score) return 1;
  return a->item < b->item ? -1 : (a->item > b->item ? 1 : 0);
}

/* Chunk index that holds sorted position pos (a plain search over the chunk starts). */
static int64_t chunk_of(int64_t pos, int64_t M, int64_t n_c) {
  int64_t c = 0;
  while (c + 1 < n_c && oracle_chunk_start(c + 1, M, n_c) <= pos) ++c;
  return c;
}

/* Steps 3-4: for every row, the candidate negatives from all rounds (window items of
 * the row's chunk, positive removed, de-duplicated) and the k best of them.
 *   permX [n_r*N], permY [n_r*C]  : per-round stable bucket orders (from above)
 *   rows [n_rows]                : the rows to compute (NULL: all N rows, n_rows = N)
 *   selected [n_rows*k]          : item ids, best first, -1 padded
 *   sel_score [n_rows*k]         : their fp32 scores (-inf for padding)
 *   n_cand [n_rows]              : number of distinct candidates of each row */
void oracle_select(const float* X, const float* Y, const int32_t* target, int64_t N, int64_t C,
                   int32_t d, int32_t n_c, int32_t n_ec, int32_t n_r, int32_t k,
                   const int32_t* permX, const int32_t* permY, const int64_t* rows,
                   int64_t n_rows, int32_t* selected, float* sel_score, int64_t* n_cand) {
  /* position of each row in each round's sorted order */
  int64_t* posX = (int64_t*)malloc(sizeof(int64_t) * (size_t)(N * n_r > 0 ? N * n_r : 1));
  for (int32_t r = 0; r < n_r; ++r)
    for (int64_t p = 0; p < N; ++p) posX[(int64_t)r * N + permX[(int64_t)r * N + p]] = p;

#pragma omp parallel
  {
    unsigned char* seen = (unsigned char*)calloc((size_t)C, 1);
    cand_t* cand = (cand_t*)malloc(sizeof(cand_t) * (size_t)C);
#pragma omp for schedule(dynamic, 16)
    for (int64_t o = 0; o < n_rows; ++o) {
      const int64_t i = rows ? rows[o] : o;
      int64_t n = 0;
      for (int32_t r = 0; r < n_r; ++r) {
        int64_t c = chunk_of(posX[(int64_t)r * N + i], N, n_c);
        int64_t c_lo = c - n_ec < 0 ? 0 : c - n_ec;
        int64_t c_hi = c + n_ec + 1 > n_c ? n_c : c + n_ec + 1;
        int64_t q_lo = oracle_chunk_start(c_lo, C, n_c);
        int64_t q_hi = oracle_chunk_start(c_hi, C, n_c);
        for (int64_t q = q_lo; q < q_hi; ++q) {
          int32_t j = permY[(int64_t)r * C + q];
          if (j == target[i] || seen[j]) continue;
          seen[j] = 1;
          cand[n].item = j;
          ++n;
        }
      }
      for (int64_t a = 0; a < n; ++a) {
        cand[a].score = dot_f32(X + i * (int64_t)d, Y + (int64_t)cand[a].item * d, d);
        seen[cand[a].item] = 0;
      }
      qsort(cand, (size_t)n, sizeof(cand_t), cmp_cand);
      for (int32_t a = 0; a < k; ++a) {
        if (a < n) {
          selected[o * (int64_t)k + a] = cand[a].item;
          sel_score[o * (int64_t)k + a] = cand[a].score;
        } else {
          selected[o * (int64_t)k + a] = -1;
          sel_score[o * (int64_t)k + a] = -INFINITY;
        }
      }
      n_cand[o] = n;
    }
    free(cand);
    free(seen);
  }
  free(posX);
}

/* Step 5, [RECE] Algorithm 1 loss lines with [SCE]'s subset: per row
 *   l+   = <x_i, y_{z_i}>,  l_ij = <x_i, y_j> for j in S_i
 *   lse  = log(exp(l+) + sum_j exp(l_ij)),  loss_i = lse - l+,  L = mean_i loss_i
 * in fp64.  selected entries < 0 are padding. */
void oracle_rece_loss(const float* X, const float* Y, const int32_t* target, int64_t N,
                      int32_t d, int32_t k, const int32_t* selected, double* row_loss,
                      double* lse, double* loss) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < N; ++i) {
    const float* x = X + i * (int64_t)d;
    double lp = dot_f64(x, Y + (int64_t)target[i] * d, d);
    double m = lp;
    for (int32_t a = 0; a < k; ++a) {
      int32_t j = selected[i * (int64_t)k + a];
      if (j < 0) continue;
      double l = dot_f64(x, Y + (int64_t)j * d, d);
      if (l > m) m = l;
    }
    double s = exp(lp - m);
    for (int32_t a = 0; a < k; ++a) {
      int32_t j = selected[i * (int64_t)k + a];
      if (j < 0) continue;
      s += exp(dot_f64(x, Y + (int64_t)j * d, d) - m);
    }
    lse[i] = m + log(s);
    row_loss[i] = lse[i] - lp;
  }
  double total = 0.0;
  for (int64_t i = 0; i < N; ++i) total += row_loss[i];
  *loss = N > 0 ? total / (double)N : 0.0;
}

/* Step 6, [RECE] equation (4) restricted to the row's positive and its selected
 * negatives (selection held constant):
 *   p_ij = exp(l_ij - lse_i),  g_ij = (p_ij - [j == z_i]) * dloss / N
 *   dX_i = sum_j g_ij y_j,     dY_j = sum_i g_ij x_i            (fp64) */
void oracle_rece_grad(const float* X, const float* Y, const int32_t* target, int64_t N, int64_t C,
                      int32_t d, int32_t k, const int32_t* selected, const double* lse,
                      double dloss, double* dX, double* dY) {
  double scale = N > 0 ? dloss / (double)N : 0.0;
  memset(dY, 0, sizeof(double) * (size_t)C * (size_t)d);
  for (int64_t i = 0; i < N; ++i) {
    const float* x = X + i * (int64_t)d;
    double* dx = dX + i * (int64_t)d;
    for (int32_t t = 0; t < d; ++t) dx[t] = 0.0;
    for (int32_t a = -1; a < k; ++a) {
      int32_t j = a < 0 ? target[i] : selected[i * (int64_t)k + a];
      if (j < 0) continue;
      const float* y = Y + (int64_t)j * d;
      double p = exp(dot_f64(x, y, d) - lse[i]);
      double g = (a < 0 ? p - 1.0 : p) * scale;
      double* dy = dY + (int64_t)j * d;
      for (int32_t t = 0; t < d; ++t) {
        dx[t] += g * (double)y[t];
        dy[t] += g * (double)x[t];
      }
    }
  }
}

/* [RECE] equation (3): full cross-entropy over the whole catalogue, in fp64. */
void oracle_full_ce_loss(const float* X, const float* Y, const int32_t* target, int64_t N,
                         int64_t C, int32_t d, double* row_loss, double* lse, double* loss) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < N; ++i) {
    const float* x = X + i * (int64_t)d;
    double m = -INFINITY;
    for (int64_t j = 0; j < C; ++j) {
      double l = dot_f64(x, Y + j * d, d);
      if (l > m) m = l;
    }
    double s = 0.0;
    for (int64_t j = 0; j < C; ++j) s += exp(dot_f64(x, Y + j * d, d) - m);
    lse[i] = m + log(s);
    row_loss[i] = lse[i] - dot_f64(x, Y + (int64_t)target[i] * d, d);
  }
  double total = 0.0;
  for (int64_t i = 0; i < N; ++i) total += row_loss[i];
  *loss = N > 0 ? total / (double)N : 0.0;
}

/* [RECE] equation (4) over the whole catalogue: g_ij = (softmax_ij - [j == z_i]) dloss/N. */
void oracle_full_ce_grad(const float* X, const float* Y, const int32_t* target, int64_t N,
                         int64_t C, int32_t d, const double* lse, double dloss, double* dX,
                         double* dY) {
  double scale = N > 0 ? dloss / (double)N : 0.0;
  memset(dY, 0, sizeof(double) * (size_t)C * (size_t)d);
  for (int64_t i = 0; i < N; ++i) {
    const float* x = X + i * (int64_t)d;
    double* dx = dX + i * (int64_t)d;
    for (int32_t t = 0; t < d; ++t) dx[t] = 0.0;
    for (int64_t j = 0; j < C; ++j) {
      const float* y = Y + j * d;
      double g = (exp(dot_f64(x, y, d) - lse[i]) - (j == target[i] ? 1.0 : 0.0)) * scale;
      double* dy = dY + j * d;
      for (int32_t t = 0; t < d; ++t) {
        dx[t] += g * (double)y[t];
        dy[t] += g * (double)x[t];
      }
    }
  }
}

/* Algorithm 1 as printed [RECE section 3], every window item a negative (no top-k),
 * over n_r rounds with the rounds paragraph's duplicate correction: a pair (i, j)
 * computed in cnt_ij of the rounds enters every round's sum as exp(l_ij - ln cnt_ij).
 * Row i's window in round r: the sorted catalogue positions of chunks c-n_ec..c+n_ec
 * (clipped) of the chunk c that holds its sorted position; its positive is left out of
 * the window sums (it enters once, as l+):
 *   lse_i  = log(exp(l+) + sum_r sum_{j in W_r(i), j != z_i} exp(l_ij - ln cnt_ij))
 *   loss_i = lse_i - l+,   L = mean_i loss_i          (fp64)
 * permX [n_r*N], permY [n_r*C]: the rounds' stable bucket orders.  rows [n_rows]: the
 * rows to compute (NULL: all N, n_rows = N); outputs are indexed by the sample, and the
 * mean is over the sample.  The gradient takes the same sample (dY sums over it). */
static void window_of(int64_t i, int32_t r, const int64_t* posX, int64_t N, int64_t C,
                      int32_t n_c, int32_t n_ec, int64_t* q_lo, int64_t* q_hi) {
  int64_t c = chunk_of(posX[(int64_t)r * N + i], N, n_c);
  int64_t c_lo = c - n_ec < 0 ? 0 : c - n_ec;
  int64_t c_hi = c + n_ec + 1 > n_c ? n_c : c + n_ec + 1;
  *q_lo = oracle_chunk_start(c_lo, C, n_c);
  *q_hi = oracle_chunk_start(c_hi, C, n_c);
}

static int64_t* positions(const int32_t* permX, int64_t N, int32_t n_r) {
  int64_t* posX = (int64_t*)malloc(sizeof(int64_t) * (size_t)(N * n_r > 0 ? N * n_r : 1));
  for (int32_t r = 0; r < n_r; ++r)
    for (int64_t p = 0; p < N; ++p) posX[(int64_t)r * N + permX[(int64_t)r * N + p]] = p;
  return posX;
}

void oracle_window_loss(const float* X, const float* Y, const int32_t* target, int64_t N,
                        int64_t C, int32_t d, int32_t n_c, int32_t n_ec, int32_t n_r,
                        const int32_t* permX, const int32_t* permY, const int64_t* rows,
                        int64_t n_rows, double* row_loss, double* lse, double* loss) {
  int64_t* posX = positions(permX, N, n_r);
#pragma omp parallel
  {
    int32_t* cnt = (int32_t*)calloc((size_t)C, sizeof(int32_t));
#pragma omp for schedule(dynamic, 16)
    for (int64_t o = 0; o < n_rows; ++o) {
      const int64_t i = rows ? rows[o] : o;
      const float* x = X + i * (int64_t)d;
      int64_t q_lo, q_hi;
      /* how many rounds compute each pair of this row */
      for (int32_t r = 0; r < n_r; ++r) {
        window_of(i, r, posX, N, C, n_c, n_ec, &q_lo, &q_hi);
        for (int64_t q = q_lo; q < q_hi; ++q) {
          int32_t j = permY[(int64_t)r * C + q];
          if (j != target[i]) ++cnt[j];
        }
      }
      double lp = dot_f64(x, Y + (int64_t)target[i] * d, d);
      double m = lp;
      for (int32_t r = 0; r < n_r; ++r) {
        window_of(i, r, posX, N, C, n_c, n_ec, &q_lo, &q_hi);
        for (int64_t q = q_lo; q < q_hi; ++q) {
          int32_t j = permY[(int64_t)r * C + q];
          if (j == target[i]) continue;
          double l = dot_f64(x, Y + (int64_t)j * d, d) - log((double)cnt[j]);
          if (l > m) m = l;
        }
      }
      double s = exp(lp - m);
      for (int32_t r = 0; r < n_r; ++r) {
        window_of(i, r, posX, N, C, n_c, n_ec, &q_lo, &q_hi);
        for (int64_t q = q_lo; q < q_hi; ++q) {
          int32_t j = permY[(int64_t)r * C + q];
          if (j == target[i]) continue;
          s += exp(dot_f64(x, Y + (int64_t)j * d, d) - log((double)cnt[j]) - m);
        }
      }
      lse[o] = m + log(s);
      row_loss[o] = lse[o] - lp;
      for (int32_t r = 0; r < n_r; ++r) {
        window_of(i, r, posX, N, C, n_c, n_ec, &q_lo, &q_hi);
        for (int64_t q = q_lo; q < q_hi; ++q) cnt[permY[(int64_t)r * C + q]] = 0;
      }
    }
    free(cnt);
  }
  free(posX);
  double total = 0.0;
  for (int64_t o = 0; o < n_rows; ++o) total += row_loss[o];
  *loss = n_rows > 0 ? total / (double)n_rows : 0.0;
}

/* Its gradients, the buckets and windows held constant: every computed copy of a pair
 * carries g = exp(l_ij - ln cnt_ij - lse_i) dloss/N, the positive (exp(l+ - lse_i) - 1)
 * dloss/N;  dX_i = sum of g y_j,  dY_j = sum of g x_i over all copies  (fp64). */
void oracle_window_grad(const float* X, const float* Y, const int32_t* target, int64_t N,
                        int64_t C, int32_t d, int32_t n_c, int32_t n_ec, int32_t n_r,
                        const int32_t* permX, const int32_t* permY, const int64_t* rows,
                        int64_t n_rows, const double* lse, double dloss, double* dX,
                        double* dY) {
  double scale = N > 0 ? dloss / (double)N : 0.0;
  int64_t* posX = positions(permX, N, n_r);
  int32_t* cnt = (int32_t*)calloc((size_t)C, sizeof(int32_t));
  memset(dY, 0, sizeof(double) * (size_t)C * (size_t)d);
  for (int64_t o = 0; o < n_rows; ++o) {
    const int64_t i = rows ? rows[o] : o;
    const float* x = X + i * (int64_t)d;
    double* dx = dX + o * (int64_t)d;
    int64_t q_lo, q_hi;
    for (int32_t r = 0; r < n_r; ++r) {
      window_of(i, r, posX, N, C, n_c, n_ec, &q_lo, &q_hi);
      for (int64_t q = q_lo; q < q_hi; ++q) {
        int32_t j = permY[(int64_t)r * C + q];
        if (j != target[i]) ++cnt[j];
      }
    }
    const float* yz = Y + (int64_t)target[i] * d;
    double gp = (exp(dot_f64(x, yz, d) - lse[o]) - 1.0) * scale;
    for (int32_t t = 0; t < d; ++t) dx[t] = gp * (double)yz[t];
    double* dyz = dY + (int64_t)target[i] * d;
    for (int32_t t = 0; t < d; ++t) dyz[t] += gp * (double)x[t];
    for (int32_t r = 0; r < n_r; ++r) {
      window_of(i, r, posX, N, C, n_c, n_ec, &q_lo, &q_hi);
      for (int64_t q = q_lo; q < q_hi; ++q) {
        int32_t j = permY[(int64_t)r * C + q];
        if (j == target[i]) continue;
        const float* y = Y + (int64_t)j * d;
        double g = exp(dot_f64(x, y, d) - log((double)cnt[j]) - lse[o]) * scale;
        double* dy = dY + (int64_t)j * d;
        for (int32_t t = 0; t < d; ++t) {
          dx[t] += g * (double)y[t];
          dy[t] += g * (double)x[t];
        }
      }
    }
    for (int32_t r = 0; r < n_r; ++r) {
      window_of(i, r, posX, N, C, n_c, n_ec, &q_lo, &q_hi);
      for (int64_t q = q_lo; q < q_hi; ++q) cnt[permY[(int64_t)r * C + q]] = 0;
    }
  }
  free(cnt);
  free(posX);
}

/* log(1 + exp(u)) without overflow: for u > 0 it is u + log(1 + exp(-u)). */
static double softplus(double u) { return u > 0.0 ? u + log1p(exp(-u)) : log1p(exp(u)); }

/* Sampled baselines, [RECE] section 2 (Related Work), equations (1) and (2).  Row i has
 * the positive z_i and n sampled negatives neg[i][0..n) (ids < 0 are padding and take no
 * part; a sample equal to the positive is a negative like any other, as the sums are
 * written):
 *   kind 0, CE-  (2):  lse_i  = log(exp(l+) + sum_j exp(l_ij)),  loss_i = lse_i - l+
 *   kind 1, BCE+ (1):  loss_i = -log sigmoid(l+) - sum_j log(1 - sigmoid(l_ij))
 *                             = softplus(-l+) + sum_j softplus(l_ij)
 * with l = <x_i, y_j> in fp64; L = mean_i loss_i.  lse is written for kind 0 only. */
void oracle_sampled_loss(int32_t kind, const float* X, const float* Y, const int32_t* target,
                         int64_t N, int32_t d, int32_t n, const int32_t* neg,
                         double* row_loss, double* lse, double* loss) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < N; ++i) {
    const float* x = X + i * (int64_t)d;
    const int32_t* ng = neg + i * (int64_t)n;
    double lp = dot_f64(x, Y + (int64_t)target[i] * d, d);
    if (kind == 0) {
      double m = lp;
      for (int32_t a = 0; a < n; ++a) {
        if (ng[a] < 0) continue;
        double l = dot_f64(x, Y + (int64_t)ng[a] * d, d);
        if (l > m) m = l;
      }
      double s = exp(lp - m);
      for (int32_t a = 0; a < n; ++a)
        if (ng[a] >= 0) s += exp(dot_f64(x, Y + (int64_t)ng[a] * d, d) - m);
      lse[i] = m + log(s);
      row_loss[i] = lse[i] - lp;
    } else {
      double r = softplus(-lp);
      for (int32_t a = 0; a < n; ++a)
        if (ng[a] >= 0) r += softplus(dot_f64(x, Y + (int64_t)ng[a] * d, d));
      row_loss[i] = r;
    }
  }
  double total = 0.0;
  for (int64_t i = 0; i < N; ++i) total += row_loss[i];
  *loss = N > 0 ? total / (double)N : 0.0;
}

/* Gradients of equations (1) and (2), the sampled negatives held constant:
 *   CE-:   g_i+ = (p_i+ - 1) dloss/N,      g_ij = p_ij dloss/N,   p = exp(l - lse_i)
 *   BCE+:  g_i+ = (sigmoid(l+) - 1) dloss/N,  g_ij = sigmoid(l_ij) dloss/N
 *   dX_i = g_i+ y_{z_i} + sum_j g_ij y_j,   dY_j = sum over the pairs naming j of g x_i
 * (a negative sampled twice contributes twice), in fp64. */
void oracle_sampled_grad(int32_t kind, const float* X, const float* Y, const int32_t* target,
                         int64_t N, int64_t C, int32_t d, int32_t n, const int32_t* neg,
                         const double* lse, double dloss, double* dX, double* dY) {
  double scale = N > 0 ? dloss / (double)N : 0.0;
  memset(dY, 0, sizeof(double) * (size_t)C * (size_t)d);
  for (int64_t i = 0; i < N; ++i) {
    const float* x = X + i * (int64_t)d;
    double* dx = dX + i * (int64_t)d;
    for (int32_t t = 0; t < d; ++t) dx[t] = 0.0;
    for (int32_t a = -1; a < n; ++a) {
      int32_t j = a < 0 ? target[i] : neg[i * (int64_t)n + a];
      if (j < 0) continue;
      const float* y = Y + (int64_t)j * d;
      double l = dot_f64(x, y, d);
      double p = kind == 0 ? exp(l - lse[i]) : 1.0 / (1.0 + exp(-l));
      double g = (a < 0 ? p - 1.0 : p) * scale;
      double* dy = dY + (int64_t)j * d;
      for (int32_t t = 0; t < d; ++t) {
        dx[t] += g * (double)y[t];
        dy[t] += g * (double)x[t];
      }
    }
  }
}

/* Exposed for the tests: the fp32 fmaf-chain score of one pair. */
float oracle_dot_f32(const float* a, const float* b, int32_t d) { return dot_f32(a, b, d); }

/* [RECE] Algorithm 1, the randn step: the random vectors B of one call of the loss,
 * drawn from (seed, step) by a counter-based stream, so that the library and this oracle,
 * each written from the stream's published definition, draw the same numbers.
 *   SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
 *   OOPSLA 2014): for state s and gamma G = 0x9E3779B97F4A7C15 the i-th output (from 0)
 *   is mix(s + (i + 1) G), where mix(z) is z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
 *   z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31 (arithmetic mod 2^64).
 *   A call's state: s = mix(mix(seed) ^ step).
 *   A uniform from an output x: u = ((x >> 11) + 1) 2^-53, in (0, 1].
 *   Box-Muller (Box and Muller, Ann. Math. Statist. 1958), pair q of elements: from
 *   u1 = u(x_2q) and u2 = u(x_2q+1), rho = sqrt(-2 ln u1), theta = 2 pi u2 (2 pi as the
 *   double 6.283185307179586), element 2q = rho cos(theta), element 2q+1 = rho sin(theta),
 *   in fp64, rounded to fp32.  Elements follow B's row-major order [n_r][n_b][d]; with an
 *   odd count the last sine is not used. */
static uint64_t splitmix_mix(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}

uint64_t oracle_splitmix64(uint64_t s, uint64_t i) {
  return splitmix_mix(s + (i + 1) * 0x9E3779B97F4A7C15ull);
}

void oracle_draw_projections(uint64_t seed, uint64_t step, int64_t count, float* B) {
  const uint64_t s = splitmix_mix(splitmix_mix(seed) ^ step);
  for (int64_t q = 0; 2 * q < count; ++q) {
    const uint64_t x1 = oracle_splitmix64(s, (uint64_t)(2 * q));
    const uint64_t x2 = oracle_splitmix64(s, (uint64_t)(2 * q + 1));
    const double u1 = (double)((x1 >> 11) + 1) * 0x1.0p-53;
    const double u2 = (double)((x2 >> 11) + 1) * 0x1.0p-53;
    const double rho = sqrt(-2.0 * log(u1));
    const double theta = 6.283185307179586 * u2;
    B[2 * q] = (float)(rho * cos(theta));
    if (2 * q + 1 < count) B[2 * q + 1] = (float)(rho * sin(theta));
  }
}
