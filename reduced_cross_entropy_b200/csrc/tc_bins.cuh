// tc_bins.cuh -- the threshold arithmetic of the exact tensor-core selection (shared by
// select_tc.cu and scores_tc.cu): distance bins of fp32 scores below an anchor, the fp32
// threshold of a cut bin, and the bound of the scores a cut leaves out.
#pragma once

#include <stdint.h>

namespace rece {
namespace tcsel {

// Distance bins.  The anchor A is the bit pattern of a value head_bins bins beyond the
// row's max m (or the max of a sample of its scores), away from zero, so that scores a
// little above a sampled m still get bins of their own.  For m >= 0 the distance of a
// score s is A - bits(s), for m < 0 it is bits(s) - A: in both cases
// key(anchor) - key(s) with key the order-preserving integer image of an fp32 value, as
// long as s lies between zero and the anchor.  Bin = min(distance >> 20, 255): 8 bins per
// binade of |s|.  Any other score (beyond the anchor, or on the far side of zero) wraps
// to a huge distance, normally the open last bin; that only misplaces the cut, since
// the emission itself compares values and the exactness check below stays sound.
struct BinMap {
  uint32_t sig, off, anchor;
};
__device__ __forceinline__ BinMap bin_map(float m, uint32_t head_bins) {
  const uint32_t H = head_bins << 20;
  const uint32_t bm = __float_as_uint(m);
  if (!(bm & 0x80000000u)) {
    const uint32_t A = bm > 0x7F7FFFFFu - H ? 0x7F7FFFFFu : bm + H;
    return BinMap{0xFFFFFFFFu, A, A};
  }
  const uint32_t A = bm - H < 0x80000000u ? 0x80000000u : bm - H;
  return BinMap{1u, 0u - A, A};
}

// The fp32 threshold t of the cut "distance < L" (L = (b* + 1) << 20): a score between
// zero and the anchor has distance < L exactly when s >= t.  -inf when every score passes.
__device__ __forceinline__ float cut_threshold(const BinMap& b, uint32_t L) {
  if (b.sig != 1u) return b.anchor >= L ? __uint_as_float(b.anchor - L + 1u) : 0.0f;
  const uint64_t tb = uint64_t(b.anchor) + L - 1u;  // L - 1 ulps beyond the anchor
  return tb < 0xFF800000ull ? __uint_as_float(uint32_t(tb)) : -INFINITY;
}

// The largest fp32 value below t (t finite or +0/-0): every score < t is <= it.
__device__ __forceinline__ float value_below(float t) {
  const uint32_t b = __float_as_uint(t);
  if (t > 0.0f) return __uint_as_float(b - 1u);
  if (t == 0.0f) return __uint_as_float(0x80000001u);
  return __uint_as_float(b + 1u);
}

}  // namespace tcsel
}  // namespace rece
