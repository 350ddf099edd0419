// select.cu -- cumulative-eta block selection and temporal union (sm_100a).
//
// Wan & Chen, "Attention Routing Stabilizes Early: Working-Set Inference for
// Recurrent-Depth Language Models": section 3 defines the support as the
// smallest set of admissible keys whose cumulative mass is at least eta;
// section 5.1 / 6.1 apply it to block masses r_qb ranked by size; appendix B
// ("WISE configuration") unions the per-step supports over the discovery
// window.  Ties in the ranking go to the lower block index.
//
// One warp per (bh, q) row.  Lane l holds the masses of blocks l, l+32, ...
// so the selected set of word s is one __ballot_sync.  Instead of sorting,
// the kernel finds the cut value tau = the largest float with
// f(tau) = sum_{b : r_b >= tau} r_b >= eta by bisection over the float bit
// patterns (masses are >= 0, so bit order equals value order and f is
// monotone for the fixed reduction tree).  Every block above tau is in the
// sorted prefix; blocks equal to tau are added in ascending index order until
// the cumulative mass reaches eta, which is exactly the shortest prefix of the
// (mass desc, index asc) ranking.

#include <cstdint>

#include "wise_internal.h"

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

template <int MAXW>
__global__ void __launch_bounds__(256)
    select_union_kernel(const float* __restrict__ mass, uint32_t* __restrict__ ubits,
                        uint32_t* __restrict__ sbits, float eta, long long rows, int nq) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;  // warp-uniform
  const int W = (nq + 31) >> 5;
  const int q = (int)(row % nq);
  const float* mrow = mass + row * (long long)nq;

  float v[MAXW];
  bool ok[MAXW];
#pragma unroll
  for (int s = 0; s < MAXW; ++s) {
    const int kb = s * 32 + lane;
    ok[s] = (s < W) && (kb <= q);
    v[s] = ok[s] ? mrow[kb] : 0.f;
  }

  bool sel[MAXW];
  const float total = warp_sum_ge<MAXW>(v, ok, 0.f);
  if (!(eta < 1.0f) || total < eta) {
#pragma unroll
    for (int s = 0; s < MAXW; ++s) sel[s] = ok[s];
  } else {
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

  uint32_t word = 0u;
#pragma unroll
  for (int s = 0; s < MAXW; ++s) {
    const uint32_t w = __ballot_sync(0xffffffffu, sel[s]);
    if (lane == s) word = w;
  }
  if (lane < W) {
    const long long at = row * W + lane;
    if (sbits != nullptr) sbits[at] = word;
    ubits[at] |= word;
  }
}

cudaError_t launch_select_union(const float* mass, uint32_t* union_bits, uint32_t* step_bits,
                                float eta, int BH, int nq, cudaStream_t stream) {
  const long long rows = (long long)BH * nq;
  const int W = (nq + 31) / 32;
  const int warps_per_block = 8;
  const unsigned grid = (unsigned)((rows + warps_per_block - 1) / warps_per_block);
  const dim3 block(32 * warps_per_block);
  if (W <= 1)
    select_union_kernel<1><<<grid, block, 0, stream>>>(mass, union_bits, step_bits, eta, rows, nq);
  else if (W <= 2)
    select_union_kernel<2><<<grid, block, 0, stream>>>(mass, union_bits, step_bits, eta, rows, nq);
  else if (W <= 4)
    select_union_kernel<4><<<grid, block, 0, stream>>>(mass, union_bits, step_bits, eta, rows, nq);
  else if (W <= 8)
    select_union_kernel<8><<<grid, block, 0, stream>>>(mass, union_bits, step_bits, eta, rows, nq);
  else if (W <= 16)
    select_union_kernel<16><<<grid, block, 0, stream>>>(mass, union_bits, step_bits, eta, rows, nq);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace wise
