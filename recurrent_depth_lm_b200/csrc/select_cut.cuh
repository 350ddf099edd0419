// select_cut.cuh -- the cumulative-eta cut of one row held by one warp.
//
// Wan & Chen, "Attention Routing Stabilizes Early: Working-Set Inference for
// Recurrent-Depth Language Models": section 3 ("attention support") and section 6.1
// define the support of a row as the shortest prefix of its blocks ranked by mass
// (descending, ties to the lower block index) whose cumulative mass reaches eta.
// Used by every selection kernel of select.cu.
//
// Arithmetic.  Each mass is clamped to [0, 1] (NaN counts as 0) and rounded to the
// nearest multiple of 2^-21; cumulative sums are then exact integer sums (a row holds
// at most 1024 masses, so no sum exceeds 2^31), the same in any order, and a prefix
// reaches eta when its sum is at least ceil(eta * 2^21).  The ranking uses the clamped
// fp32 masses themselves.
//
// Method.  Lane l holds the masses of blocks s * 32 + l.  The cut value tau (the
// smallest mass of the shortest prefix) is found by a most-significant-digit radix
// select over the bit patterns of the masses (non-negative floats order like their
// bits): four passes over 8-bit digits, each building a histogram of integer mass
// per digit in shared memory, among the blocks that match the digits found so far,
// and taking the highest digit at which the mass above plus the digit's mass reaches
// the target.  Blocks above tau are kept; blocks equal to tau are added in ascending
// index order until the sum reaches the target.

#pragma once

#include <cstdint>

namespace wise {

constexpr float kCutScale = 2097152.0f;   // 2^21 units per unit of mass

__device__ __forceinline__ float cut_clamp(float r) {
  return fminf(fmaxf(r, 0.f), 1.f);     // fmaxf(NaN, 0) = 0
}

__device__ __forceinline__ uint32_t cut_units(float r) {
  return __float2uint_rn(cut_clamp(r) * kCutScale);
}

// Shortest prefix of the (mass desc, index asc) ranking whose sum in units reaches
// `target`, for the masses v[s] of blocks s * 32 + lane that have ok[s] set.  Requires
// 0 < target <= the row's total in units.  hist: 256 words of shared memory owned by
// this warp, 16-byte aligned.  All 32 lanes must call.
template <int MAXW>
__device__ __forceinline__ void cut_at(const float (&v)[MAXW], const bool (&ok)[MAXW],
                                       uint32_t target, int lane, bool (&sel)[MAXW],
                                       uint32_t* hist) {
  uint32_t key[MAXW], u[MAXW];
#pragma unroll
  for (int s = 0; s < MAXW; ++s) {
    key[s] = __float_as_uint(cut_clamp(v[s])) & 0x7fffffffu;   // -0 ranks as +0
    u[s] = ok[s] ? cut_units(v[s]) : 0u;
  }
  uint32_t prefix = 0u;   // digits of tau found so far
  uint32_t above = 0u;    // mass of the blocks whose key is above every key with that prefix
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    reinterpret_cast<uint4*>(hist)[2 * lane] = make_uint4(0u, 0u, 0u, 0u);
    reinterpret_cast<uint4*>(hist)[2 * lane + 1] = make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
#pragma unroll
    for (int s = 0; s < MAXW; ++s) {
      const bool in = u[s] != 0u && (pass == 0 || (key[s] >> (shift + 8)) == prefix);
      if (in) atomicAdd(&hist[(key[s] >> shift) & 255u], u[s]);
    }
    __syncwarp();
    // lane L takes digits 255 - 8 L - i, i = 0..7: the warp walks the digits downwards
    const uint4 hi4 = reinterpret_cast<const uint4*>(hist)[2 * (31 - lane) + 1];
    const uint4 lo4 = reinterpret_cast<const uint4*>(hist)[2 * (31 - lane)];
    const uint32_t h[8] = {hi4.w, hi4.z, hi4.y, hi4.x, lo4.w, lo4.z, lo4.y, lo4.x};
    uint32_t c[8];
    uint32_t run = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      run += h[i];
      c[i] = run;
    }
    uint32_t x = run;   // inclusive scan of the lane totals, lane 0 first
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const uint32_t before = above + x - run;   // mass of all higher digits' lanes
    int first = 8;
#pragma unroll
    for (int i = 7; i >= 0; --i)
      if (before + c[i] >= target) first = i;
    uint32_t rest = 0u;   // mass above the chosen digit
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i == first) rest = before + c[i] - h[i];
    // The previous pass (or the total) guarantees that some digit reaches the target.
    const int lsel = __ffs(__ballot_sync(0xffffffffu, first < 8)) - 1;
    const int digit_i = __shfl_sync(0xffffffffu, first, lsel);
    above = __shfl_sync(0xffffffffu, rest, lsel);
    prefix = (prefix << 8) | (uint32_t)(255 - 8 * lsel - digit_i);
    __syncwarp();   // every lane has read hist before the next pass clears it
  }
  const uint32_t tau = prefix;
  uint32_t running = above;   // mass strictly above tau
#pragma unroll
  for (int s = 0; s < MAXW; ++s) sel[s] = ok[s] && key[s] > tau;
#pragma unroll
  for (int s = 0; s < MAXW; ++s) {
    uint32_t ties = __ballot_sync(0xffffffffu, ok[s] && key[s] == tau);
    const uint32_t ut = __shfl_sync(0xffffffffu, u[s], ties ? __ffs(ties) - 1 : 0);
    while (ties != 0u && running < target) {
      const int b = __ffs(ties) - 1;
      ties &= ties - 1u;
      running += ut;
      if (lane == b) sel[s] = true;
    }
  }
}

// Shortest prefix of the (mass desc, index asc) ranking with cumulative mass >= eta.
// If eta >= 1, or the whole row does not reach eta, every admissible block is kept.
template <int MAXW>
__device__ __forceinline__ void eta_cut(const float (&v)[MAXW], const bool (&ok)[MAXW], float eta,
                                        int lane, bool (&sel)[MAXW], uint32_t* hist) {
  uint32_t part = 0u;
#pragma unroll
  for (int s = 0; s < MAXW; ++s) part += ok[s] ? cut_units(v[s]) : 0u;
  const uint32_t total = __reduce_add_sync(0xffffffffu, part);
  const uint32_t target = (uint32_t)ceilf(fminf(eta, 1.0f) * kCutScale);
  if (!(eta < 1.0f) || total < target || target == 0u) {
#pragma unroll
    for (int s = 0; s < MAXW; ++s) sel[s] = ok[s];
    return;
  }
  cut_at<MAXW>(v, ok, target, lane, sel, hist);
}

}  // namespace wise
