// mass.cu -- block mass from per-(row, key block) log-sum-exps (one-pass window steps).
//
// Wan & Chen, "Attention Routing Stabilizes Early: Working-Set Inference for
// Recurrent-Depth Language Models", section 5.1: r_qb = (1/|I_q|) sum_{i in I_q}
// sum_{j in I_b} A_ij.  The dense attention kernel, while it runs, records for
// every row i and admissible key block b the block's log2-sum-exp
// blse_ib = log2 sum_{j in I_b, j <= i} 2^(s_ij * scale * log2 e); with the row's
// final normaliser lse_i the inner sum is 2^(blse_ib - lse_i * log2 e).  This
// kernel does the outer mean: one warp per (bh, q), lane = row of the query
// block, a butterfly sum per key block.

#include <cstdint>

#include "sm100.cuh"
#include "wise_internal.h"

namespace wise {

__global__ void __launch_bounds__(256)
    mass_from_blse_kernel(const float* __restrict__ blse, const float* __restrict__ lse,
                          float* __restrict__ mass, long long rows, int n, int nq) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;  // warp-uniform
  const long long bh = row / nq;
  const int q = (int)(row % nq);
  const int i = q * 32 + lane;
  const float l2 = lse[bh * n + i] * 1.4426950408889634f;
  const float* src = blse + bh * (long long)nq * n + i;
  float* dst = mass + (bh * nq + q) * (long long)nq;
  // four key blocks per round: independent butterflies
  for (int b0 = 0; b0 <= q; b0 += 4) {
    float v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int b = b0 + u;
      v[u] = b <= q ? fast_exp2(src[(long long)b * n] - l2) : 0.f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] += __shfl_xor_sync(0xffffffffu, v[u], o);
    }
    if (lane < 4 && b0 + lane <= q) {
      float mine = v[0];
#pragma unroll
      for (int u = 1; u < 4; ++u)
        if (lane == u) mine = v[u];
      dst[b0 + lane] = mine * (1.0f / 32.0f);
    }
  }
}

cudaError_t launch_mass_from_blse(const float* blse, const float* lse, float* mass, int BH,
                                  int n, cudaStream_t stream) {
  const int nq = n / 32;
  const long long rows = (long long)BH * nq;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  mass_from_blse_kernel<<<grid, 256, 0, stream>>>(blse, lse, mass, rows, n, nq);
  return cudaGetLastError();
}

}  // namespace wise
