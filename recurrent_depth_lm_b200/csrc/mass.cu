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
constexpr int kGroupRows = 256;            // rows per item (two 128-row halves)
constexpr int kChunk = 4;                  // key blocks per item
constexpr int kWarps = 8;                  // warps (items) per CTA
constexpr float kLog2e = 1.4426950408889634f;
}  // namespace

// RB = block size in tokens (32, or 16 for the 16-token blocks).  A group of 256 rows holds
// G = 256 / RB row blocks; group g needs key blocks 0 .. G (g + 1) - 1 (those at or before
// its last 32-token diagonal block), i.e. G (g + 1) / kChunk items; groups 0 .. g - 1 hold
// (G / kChunk) g (g + 1) / 2.  Key block kb is admissible for row block q when kb <= q at
// RB = 32, and when kb / 2 <= q / 2 at RB = 16 (the diagonal 32-block's upper 16 x 16
// quarter has blse = -inf, so its mass comes out 0, as the 16-token mass defines).
template <int RB>
__global__ void __launch_bounds__(kWarps * 32)
    block_mass_kernel(const float* __restrict__ blse, const float* __restrict__ lse,
                      float* __restrict__ mass, int n, int nb, long long items_per_bh,
                      long long items) {
  constexpr int G = kGroupRows / RB;          // row blocks per group
  constexpr int kPerGroupRow = G / kChunk;    // items per group per group index
  constexpr int kLanesPerBlock = RB / 4;      // lanes holding one row block (4 rows each)
  const int lane = threadIdx.x & 31;
  const long long item = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (item >= items) return;   // warp-uniform
  const long long bh = item / items_per_bh;
  const int it = (int)(item % items_per_bh);
  int g = (int)((sqrtf(8.0f * (float)it / kPerGroupRow + 1.0f) - 1.0f) * 0.5f);
  while (g > 0 && kPerGroupRow * g * (g + 1) / 2 > it) --g;
  while (kPerGroupRow * (g + 1) * (g + 2) / 2 <= it) ++g;
  const int c = it - kPerGroupRow * g * (g + 1) / 2;
  const int q0 = g * G;
  const int nrow = min(G, nb - q0);
  const int kb0 = c * kChunk;
  const int qlast = q0 + nrow - 1;
  const int kb_lim = RB == 32 ? qlast + 1 : (qlast | 1) + 1;
  const int kb_end = min(kb0 + kChunk, kb_lim);   // key blocks kb0 .. kb_end - 1

  // This lane's rows: 4 (lane % (RB/4)) .. + 3 of row block qa[h] = q0 + (128 / RB) h + lane / (RB/4).
  int qa[2];
  float4 l4[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    qa[h] = q0 + (128 / RB) * h + lane / kLanesPerBlock;
    l4[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (qa[h] < q0 + nrow)
      l4[h] = __ldg(reinterpret_cast<const float4*>(lse + bh * n + (long long)q0 * RB +
                                                    128 * h + 4 * lane));
    else
      qa[h] = -1;   // past the last row block: never admissible
  }
  auto admissible = [&](int kb, int q) {
    return q >= 0 && (RB == 32 ? kb <= q : (kb >> 1) <= (q >> 1));
  };
  const float* base = blse + bh * nb * (long long)n + (long long)q0 * RB + 4 * lane;
  float4 x[kChunk][2];
#pragma unroll
  for (int u = 0; u < kChunk; ++u) {
    const int kb = kb0 + u;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      x[u][h] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (kb < kb_end && admissible(kb, qa[h]))
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
      if (admissible(kb, qa[h])) {
        const float4 y = x[u][h];
        a = (fast_exp2(fmaf(-l4[h].x, kLog2e, y.x)) + fast_exp2(fmaf(-l4[h].y, kLog2e, y.y))) +
            (fast_exp2(fmaf(-l4[h].z, kLog2e, y.z)) + fast_exp2(fmaf(-l4[h].w, kLog2e, y.w)));
      }
#pragma unroll
      for (int o = 1; o < kLanesPerBlock; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      part[h] = a;
    }
    if ((lane & (kLanesPerBlock - 1)) == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h)
        if (admissible(kb, qa[h]))
          mass[(bh * nb + qa[h]) * (long long)nb + kb] = part[h] * (1.0f / RB);
    }
  }
}

template <int RB>
static cudaError_t launch_mass_rb(const float* blse, const float* lse, float* mass, int BH, int n,
                                  cudaStream_t stream) {
  constexpr int G = kGroupRows / RB;
  const int nb = n / RB;
  const long long groups = (nb + G - 1) / G;
  const long long items_per_bh = (G / kChunk) * groups * (groups + 1) / 2;
  const long long items = items_per_bh * BH;
  const long long ctas = (items + kWarps - 1) / kWarps;
  if (ctas > 0x7fffffffLL) return cudaErrorInvalidValue;
  block_mass_kernel<RB><<<(unsigned)ctas, kWarps * 32, 0, stream>>>(blse, lse, mass, n, nb,
                                                                   items_per_bh, items);
  return cudaGetLastError();
}

cudaError_t launch_block_mass(const float* blse, const float* lse, float* mass, int BH, int n,
                              cudaStream_t stream) {
  return launch_mass_rb<32>(blse, lse, mass, BH, n, stream);
}

cudaError_t launch_block_mass16(const float* blse16, const float* lse, float* mass16, int BH,
                                int n, cudaStream_t stream) {
  return launch_mass_rb<16>(blse16, lse, mass16, BH, n, stream);
}

}  // namespace wise
