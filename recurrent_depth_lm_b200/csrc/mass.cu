// mass.cu -- block mass from per-(row, key block) log-sum-exps (one-pass window steps).
//
// Wan & Chen, "Attention Routing Stabilizes Early: Working-Set Inference for
// Recurrent-Depth Language Models", section 5.1: r_qb = (1/|I_q|) sum_{i in I_q}
// sum_{j in I_b} A_ij.  The dense attention kernel, while it runs, records for
// every row i and admissible key block b the block's log2-sum-exp
// blse_ib = log2 sum_{j in I_b, j <= i} 2^(s_ij * scale * log2 e); with the row's
// final normaliser lse_i the inner sum is 2^(blse_ib - lse_i * log2 e).  This
// kernel does the outer mean: one warp per (bh, q); lane l takes key blocks l,
// l + 32, ... of the row and reads that block's 32 consecutive row values (blse is
// [bh][key block][row]) as eight 16-byte loads, then sums them on its own, so a
// warp keeps 4 KB of loads in flight and writes 128 consecutive bytes of mass.

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
  // log2-domain lse of the 32 rows of block q, every lane holding all 32
  const float mine = lse[bh * n + q * 32 + lane] * 1.4426950408889634f;
  float l2[32];
#pragma unroll
  for (int r = 0; r < 32; ++r) l2[r] = __shfl_sync(0xffffffffu, mine, r);
  const float* base = blse + bh * (long long)nq * n + q * 32;
  float* dst = mass + (bh * nq + q) * (long long)nq;
  for (int b = lane; b <= q; b += 32) {
    const float4* src = reinterpret_cast<const float4*>(base + (long long)b * n);
    float4 x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = __ldg(src + u);
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      a0 += fast_exp2(x[u].x - l2[4 * u]) + fast_exp2(x[u].y - l2[4 * u + 1]);
      a1 += fast_exp2(x[u].z - l2[4 * u + 2]) + fast_exp2(x[u].w - l2[4 * u + 3]);
    }
    dst[b] = (a0 + a1) * (1.0f / 32.0f);
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
