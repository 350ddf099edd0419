// mass.cu -- block mass from per-(row, key block) log-sum-exps (one-pass window steps).
//
// Wan & Chen, "Attention Routing Stabilizes Early: Working-Set Inference for
// Recurrent-Depth Language Models", section 5.1: r_qb = (1/|I_q|) sum_{i in I_q}
// sum_{j in I_b} A_ij.  The dense attention kernel, while it runs, records for
// every row i and admissible key block b the block's log2-sum-exp
// blse_ib = log2 sum_{j in I_b, j <= i} 2^(s_ij * scale * log2 e); with the row's
// final normaliser lse_i the inner sum is 2^(blse_ib - lse_i * log2 e).  This
// kernel does the outer mean.
//
// blse is [bh][key block][row], so for one key block the 256 rows of eight
// consecutive query blocks are 1 KB of contiguous memory.  One warp takes one work
// item: a (bh, group of eight query blocks, chunk of kChunk key blocks) tile of the
// causal triangle.  Each lane issues all of the item's loads first (two 16-byte loads
// per key block: rows 4 l .. 4 l + 3 of the group's first and second 128 rows), then
// the eight lanes holding one query block's 32 rows sum them with three shuffles.
// Items are numbered group by group, so every warp of the grid has the same short
// chain of work (one round of loads) and the grid streams the causal triangle in about
// two waves of resident warps at 4K.  Only admissible (row block, key block) pairs are
// read or written.

#include <cstdint>

#include "sm100.cuh"
#include "wise_internal.h"

namespace wise {

namespace {
constexpr int kGroup = 8;                  // query blocks per item
constexpr int kChunk = 4;                  // key blocks per item
constexpr int kPerGroupRow = kGroup / kChunk;
constexpr int kWarps = 8;                  // warps (items) per CTA
constexpr float kLog2e = 1.4426950408889634f;
}  // namespace

// Items of one bh: group g (query blocks 8 g .. 8 g + 7) has kPerGroupRow * (g + 1) chunks,
// covering key blocks 0 .. 8 g + 7; groups 0 .. g - 1 hold kPerGroupRow * g (g + 1) / 2.
__global__ void __launch_bounds__(kWarps * 32)
    block_mass_kernel(const float* __restrict__ blse, const float* __restrict__ lse,
                      float* __restrict__ mass, int n, int nq, long long items_per_bh,
                      long long items) {
  const int lane = threadIdx.x & 31;
  const long long item = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (item >= items) return;   // warp-uniform
  const long long bh = item / items_per_bh;
  const int it = (int)(item % items_per_bh);
  int g = (int)((sqrtf(8.0f * (float)it / kPerGroupRow + 1.0f) - 1.0f) * 0.5f);
  while (g > 0 && kPerGroupRow * g * (g + 1) / 2 > it) --g;
  while (kPerGroupRow * (g + 1) * (g + 2) / 2 <= it) ++g;
  const int c = it - kPerGroupRow * g * (g + 1) / 2;
  const int q0 = g * kGroup;
  const int nrow = min(kGroup, nq - q0);
  const int kb0 = c * kChunk;
  const int kb_end = min(kb0 + kChunk, q0 + nrow);   // key blocks kb0 .. kb_end - 1

  // This lane's rows: 4 (lane % 8) .. + 3 of query block qa[h] = q0 + 4 h + lane / 8.
  int qa[2];
  float4 l4[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    qa[h] = q0 + 4 * h + (lane >> 3);
    l4[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (qa[h] < q0 + nrow)
      l4[h] = __ldg(reinterpret_cast<const float4*>(lse + bh * n + (long long)q0 * 32 +
                                                    128 * h + 4 * lane));
    else
      qa[h] = -1;   // past the last query block: never admissible
  }
  const float* base = blse + bh * nq * (long long)n + (long long)q0 * 32 + 4 * lane;
  float4 x[kChunk][2];
#pragma unroll
  for (int u = 0; u < kChunk; ++u) {
    const int kb = kb0 + u;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      x[u][h] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (kb < kb_end && qa[h] >= kb)
        x[u][h] = __ldg(reinterpret_cast<const float4*>(base + (long long)kb * n + 128 * h));
    }
  }
#pragma unroll
  for (int u = 0; u < kChunk; ++u) {
    const int kb = kb0 + u;
    if (kb >= kb_end) break;   // warp-uniform
    float part[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float a = 0.f;
      if (qa[h] >= kb) {
        const float4 y = x[u][h];
        a = (fast_exp2(fmaf(-l4[h].x, kLog2e, y.x)) + fast_exp2(fmaf(-l4[h].y, kLog2e, y.y))) +
            (fast_exp2(fmaf(-l4[h].z, kLog2e, y.z)) + fast_exp2(fmaf(-l4[h].w, kLog2e, y.w)));
      }
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      a += __shfl_xor_sync(0xffffffffu, a, 4);
      part[h] = a;
    }
    if ((lane & 7) == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h)
        if (qa[h] >= kb) mass[(bh * nq + qa[h]) * (long long)nq + kb] = part[h] * (1.0f / 32.0f);
    }
  }
}

cudaError_t launch_block_mass(const float* blse, const float* lse, float* mass, int BH, int n,
                              cudaStream_t stream) {
  const int nq = n / 32;
  const long long groups = (nq + kGroup - 1) / kGroup;
  const long long items_per_bh = kPerGroupRow * groups * (groups + 1) / 2;
  const long long items = items_per_bh * BH;
  const long long ctas = (items + kWarps - 1) / kWarps;
  if (ctas > 0x7fffffffLL) return cudaErrorInvalidValue;
  block_mass_kernel<<<(unsigned)ctas, kWarps * 32, 0, stream>>>(blse, lse, mass, n, nq,
                                                               items_per_bh, items);
  return cudaGetLastError();
}

}  // namespace wise
