// select_cut.cuh -- the cumulative-eta cut of one row held by one warp.
//
// Wan & Chen, "Attention Routing Stabilizes Early: Working-Set Inference for
// Recurrent-Depth Language Models": section 3 ("attention support") and section 6.1
// define the support of a row as the shortest prefix of its blocks ranked by mass
// (descending, ties to the lower block index) whose cumulative mass reaches eta.
// Used by the selection kernels (select.cu) and the fused block-mass selection
// (mass.cu), so both give the same bits for the same fp32 masses.
//
// Lane l holds the masses v[s] of blocks s * 32 + l.  Instead of sorting, the cut
// value tau = the largest float with f(tau) = sum_{b : r_b >= tau} r_b >= eta is
// found by bisection over the float bit patterns (masses are >= 0, so bit order
// equals value order and f is monotone for the fixed reduction tree).  Every block
// above tau is in the sorted prefix; blocks equal to tau are added in ascending
// index order until the cumulative mass reaches eta.

#pragma once

#include <cstdint>

namespace wise {

template <int MAXW>
__device__ __forceinline__ float warp_sum_ge(const float (&v)[MAXW], const bool (&ok)[MAXW],
                                             float tau) {
  float a = 0.f;
#pragma unroll
  for (int s = 0; s < MAXW; ++s) a += (ok[s] && v[s] >= tau) ? v[s] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
  return a;
}

// Shortest prefix of the (mass desc, index asc) ranking with cumulative mass >= eta,
// for the masses v[s] of blocks s * 32 + lane that have ok[s] set.
template <int MAXW>
__device__ __forceinline__ void eta_cut(const float (&v)[MAXW], const bool (&ok)[MAXW], float eta,
                                        int lane, bool (&sel)[MAXW]) {
  const float total = warp_sum_ge<MAXW>(v, ok, 0.f);
  if (!(eta < 1.0f) || total < eta) {
#pragma unroll
    for (int s = 0; s < MAXW; ++s) sel[s] = ok[s];
    return;
  }
  // invariant: f(lo) >= eta, f(hi) < eta
  uint32_t lo = 0u, hi = 0x7F800000u;
  while (hi - lo > 1u) {
    const uint32_t mid = lo + ((hi - lo) >> 1);
    if (warp_sum_ge<MAXW>(v, ok, __uint_as_float(mid)) >= eta)
      lo = mid;
    else
      hi = mid;
  }
  const float tau = __uint_as_float(lo);
  float running = warp_sum_ge<MAXW>(v, ok, __uint_as_float(hi));  // mass strictly above tau
#pragma unroll
  for (int s = 0; s < MAXW; ++s) sel[s] = ok[s] && v[s] > tau;
#pragma unroll
  for (int s = 0; s < MAXW; ++s) {
    uint32_t ties = __ballot_sync(0xffffffffu, ok[s] && v[s] == tau);
    while (ties != 0u && running < eta) {
      const int b = __ffs(ties) - 1;
      ties &= ties - 1u;
      running += tau;
      if (lane == b) sel[s] = true;
    }
  }
}

}  // namespace wise
