// mass.cu -- block mass from per-(row, key block) log-sum-exps, and the window step's
// selection on the same rows (one-pass window steps).
//
// Wan & Chen, "Attention Routing Stabilizes Early: Working-Set Inference for
// Recurrent-Depth Language Models", section 5.1: r_qb = (1/|I_q|) sum_{i in I_q}
// sum_{j in I_b} A_ij.  The dense attention kernel, while it runs, records for
// every row i and admissible key block b the block's log2-sum-exp
// blse_ib = log2 sum_{j in I_b, j <= i} 2^(s_ij * scale * log2 e); with the row's
// final normaliser lse_i the inner sum is 2^(blse_ib - lse_i * log2 e).  This
// kernel does the outer mean.
//
// One CTA per (bh, group of eight query blocks).  blse is [bh][key block][row], so
// for one key block the group's 256 rows are 1 KB of contiguous memory: warp w takes
// key blocks w, w + 8, ..., and each lane makes two 16-byte loads per key block
// (rows 4 l .. 4 l + 3 of the group's first and second 128 rows); the eight lanes
// that hold one query block's 32 rows sum them with three shuffles.  Only admissible
// (row block, key block) pairs are read.  The group's mass rows collect in shared
// memory; then warp j owns query block q0 + j: it writes that row of masses
// (coalesced) and, in a window step, cuts the row at eta (section 3 "attention
// support", section 6.1; eta_cut, as in select.cu) and ORs the support into the
// working set (appendix B, "WISE configuration").

#include <cstdint>

#include "select_cut.cuh"
#include "sm100.cuh"
#include "wise_internal.h"

namespace wise {

namespace {
constexpr int kGroup = 8;   // query blocks per CTA, one warp each
constexpr float kLog2e = 1.4426950408889634f;
}  // namespace

template <int MAXW>
__global__ void __launch_bounds__(kGroup * 32)
    mass_select_kernel(const float* __restrict__ blse, const float* __restrict__ lse,
                       float* __restrict__ mass, uint32_t* __restrict__ ubits,
                       uint32_t* __restrict__ sbits, float eta, int n, int nq, int groups) {
  extern __shared__ float rows_s[];   // [kGroup][nq] masses of the group's rows
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bh = blockIdx.x / groups;
  const int q0 = (int)(blockIdx.x % groups) * kGroup;
  const int nrow = min(kGroup, nq - q0);

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
  const int kb_end = q0 + nrow;
#pragma unroll 2
  for (int kb = warp; kb < kb_end; kb += kGroup) {   // warp-uniform trip count
    const float* src = base + (long long)kb * n;
    float part[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float a = 0.f;
      if (qa[h] >= kb) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(src + 128 * h));
        a = (fast_exp2(fmaf(-l4[h].x, kLog2e, x.x)) + fast_exp2(fmaf(-l4[h].y, kLog2e, x.y))) +
            (fast_exp2(fmaf(-l4[h].z, kLog2e, x.z)) + fast_exp2(fmaf(-l4[h].w, kLog2e, x.w)));
      }
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      a += __shfl_xor_sync(0xffffffffu, a, 4);
      part[h] = a;
    }
    if ((lane & 7) == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h)
        if (qa[h] >= kb) rows_s[(qa[h] - q0) * nq + kb] = part[h] * (1.0f / 32.0f);
    }
  }
  __syncthreads();
  if (warp >= nrow) return;   // warp-uniform

  const int q = q0 + warp;
  const long long row = bh * nq + q;
  const float* srow = rows_s + warp * nq;
  float* mrow = mass + row * nq;
  for (int kb = lane; kb <= q; kb += 32) mrow[kb] = srow[kb];
  if (ubits == nullptr) return;

  const int W = (nq + 31) >> 5;
  float v[MAXW];
  bool ok[MAXW];
#pragma unroll
  for (int s = 0; s < MAXW; ++s) {
    const int kb = s * 32 + lane;
    ok[s] = (s < W) && (kb <= q);
    v[s] = ok[s] ? srow[kb] : 0.f;
  }
  bool sel[MAXW];
  eta_cut<MAXW>(v, ok, eta, lane, sel);
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

cudaError_t launch_mass_select(const float* blse, const float* lse, float* mass,
                               uint32_t* union_bits, uint32_t* step_bits, float eta, int BH,
                               int n, cudaStream_t stream) {
  const int nq = n / 32;
  const int W = (nq + 31) / 32;
  const int groups = (nq + kGroup - 1) / kGroup;
  const long long ctas = (long long)BH * groups;
  if (ctas > 0x7fffffffLL) return cudaErrorInvalidValue;
  const size_t smem = (size_t)kGroup * nq * sizeof(float);
  const dim3 grid((unsigned)ctas), block(kGroup * 32);
#define WISE_MASS_SELECT(MW)                                                                 \
  mass_select_kernel<MW><<<grid, block, smem, stream>>>(blse, lse, mass, union_bits, step_bits, \
                                                       eta, n, nq, groups)
  if (W <= 1)
    WISE_MASS_SELECT(1);
  else if (W <= 2)
    WISE_MASS_SELECT(2);
  else if (W <= 4)
    WISE_MASS_SELECT(4);
  else if (W <= 8)
    WISE_MASS_SELECT(8);
  else if (W <= 16)
    WISE_MASS_SELECT(16);
  else
    return cudaErrorInvalidValue;
#undef WISE_MASS_SELECT
  return cudaGetLastError();
}

}  // namespace wise
