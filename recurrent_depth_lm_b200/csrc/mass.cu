// mass.cu -- block mass from per-(row, key block) log-sum-exps (one-pass window steps).
//
// Wan & Chen, "Attention Routing Stabilizes Early: Working-Set Inference for
// Recurrent-Depth Language Models", section 5.1: r_qb = (1/|I_q|) sum_{i in I_q}
// sum_{j in I_b} A_ij.  The dense attention kernel, while it runs, records for
// every row i and admissible key block b the block's log2-sum-exp
// blse_ib = log2 sum_{j in I_b, j <= i} 2^(s_ij * scale * log2 e); with the row's
// final normaliser lse_i the inner sum is 2^(blse_ib - lse_i * log2 e).  This
// kernel does the outer mean.  Each warp takes one query block q and 32 of its
// key blocks (grid y = which 32): lane l reads key block b = 32 y + l's 32
// consecutive row values (blse is [bh][key block][row]) as eight 16-byte loads
// and sums them on its own, so every load of the launch is independent and the
// whole grid's loads can be in flight at once; the 32 lse values of block q are
// one broadcast row.  The warp writes 128 consecutive bytes of mass.

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
  const int b = (int)blockIdx.y * 32 + lane;
  if ((int)blockIdx.y * 32 > q) return;  // warp-uniform: no admissible block here
  if (b > q) return;
  // log2-domain lse of the 32 rows of block q (the same 128 bytes for every lane)
  const float4* lp = reinterpret_cast<const float4*>(lse + bh * n + q * 32);
  const float4* src = reinterpret_cast<const float4*>(blse + (bh * nq + b) * (long long)n + q * 32);
  float4 x[8], l[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    x[u] = __ldg(src + u);
    l[u] = __ldg(lp + u);
  }
  constexpr float kLog2e = 1.4426950408889634f;
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    a0 += fast_exp2(x[u].x - l[u].x * kLog2e) + fast_exp2(x[u].y - l[u].y * kLog2e);
    a1 += fast_exp2(x[u].z - l[u].z * kLog2e) + fast_exp2(x[u].w - l[u].w * kLog2e);
  }
  mass[(bh * nq + q) * (long long)nq + b] = (a0 + a1) * (1.0f / 32.0f);
}

cudaError_t launch_mass_from_blse(const float* blse, const float* lse, float* mass, int BH,
                                  int n, cudaStream_t stream) {
  const int nq = n / 32;
  const long long rows = (long long)BH * nq;
  const dim3 grid((unsigned)((rows + 7) / 8), (unsigned)((nq + 31) / 32));
  mass_from_blse_kernel<<<grid, 256, 0, stream>>>(blse, lse, mass, rows, n, nq);
  return cudaGetLastError();
}

}  // namespace wise
