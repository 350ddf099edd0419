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
// so the selected set of word s is one __ballot_sync; the cut itself
// (a radix select with exact fixed-point sums, then ties in index order) is
// eta_cut in select_cut.cuh.

#include <cstdint>
#include <type_traits>

#include "select_cut.cuh"
#include "wise_internal.h"

namespace wise {

template <int MAXW>
__global__ void __launch_bounds__(256)
    select_union_kernel(const float* __restrict__ mass, uint32_t* __restrict__ ubits,
                        uint32_t* __restrict__ sbits, float eta, long long rows, int nq) {
  __shared__ __align__(16) uint32_t hist_s[8][256];   // eta_cut's digit histogram, per warp
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
  eta_cut<MAXW>(v, ok, eta, lane, sel, hist_s[threadIdx.x >> 5]);

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

// Block-size variant (WISE paper appendix C.6, "Block-Size Tradeoff"): selection on
// blocks of F x 32 tokens, run as exact 32 x 32 subtiles.  One warp per coarse row (bh, Q).  The coarse mass
// is the pooled fine mass, R_QB = (1/F) sum_{q in Q} sum_{b in B, b <= q} r_qb, which
// is the block-mass definition at block size 32F.  After the cut, fine row
// q = Q F + a keeps fine block b iff coarse block b / F was kept and b <= q.
// Fine masks are written in the fine [nq, W] layout, so the schedule builder and the
// sparse kernel run unchanged.
template <int MAXWC, int F>
__global__ void __launch_bounds__(256)
    select_union_pooled_kernel(const float* __restrict__ mass, uint32_t* __restrict__ ubits,
                               uint32_t* __restrict__ sbits, float eta, long long crows, int nq) {
  __shared__ __align__(16) uint32_t hist_s[8][256];   // eta_cut's digit histogram, per warp
  const int lane = threadIdx.x & 31;
  const long long crow = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (crow >= crows) return;  // warp-uniform
  const int nQ = nq / F;
  const long long bh = crow / nQ;
  const int Q = (int)(crow % nQ);
  const int Wc = (nQ + 31) >> 5;
  const int W = (nq + 31) >> 5;
  const float* mrow = mass + (bh * nq + (long long)Q * F) * nq;  // fine row Q F

  float v[MAXWC];
  bool ok[MAXWC];
#pragma unroll
  for (int s = 0; s < MAXWC; ++s) {
    const int cb = s * 32 + lane;
    ok[s] = (s < Wc) && (cb <= Q);
    float acc = 0.f;
    if (ok[s]) {
#pragma unroll
      for (int a = 0; a < F; ++a)
#pragma unroll
        for (int c = 0; c < F; ++c)
          if (cb * F + c <= Q * F + a) acc += mrow[(long long)a * nq + cb * F + c];
    }
    v[s] = acc * (1.0f / F);
  }

  bool sel[MAXWC];
  eta_cut<MAXWC>(v, ok, eta, lane, sel, hist_s[threadIdx.x >> 5]);

  // Fine word w covers fine blocks 32w .. 32w+31 = coarse blocks 32w/F .. (32w+31)/F,
  // all in coarse slot w / F; lane i's bit is the kept flag of coarse block (32w+i)/F.
  uint32_t word = 0u;
#pragma unroll
  for (int w = 0; w < MAXWC * F; ++w) {
    const int c = (32 * w + lane) / F;
    const bool bit = __shfl_sync(0xffffffffu, (int)sel[w / F], c & 31) != 0;
    const uint32_t m = __ballot_sync(0xffffffffu, bit);
    if (lane == w) word = m;
  }
  if (lane < W) {
#pragma unroll
    for (int a = 0; a < F; ++a) {
      const int q = Q * F + a;
      const int first = 32 * lane;  // fine block of bit 0 of this word
      uint32_t clip;
      if (first > q)
        clip = 0u;
      else if (q - first >= 31)
        clip = 0xffffffffu;
      else
        clip = (2u << (q - first)) - 1u;
      const uint32_t out = word & clip;
      const long long at = (bh * nq + q) * W + lane;
      if (sbits != nullptr) sbits[at] = out;
      ubits[at] |= out;
    }
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
  else if (W <= 32)  // 16-token blocks at n = 16384
    select_union_kernel<32><<<grid, block, 0, stream>>>(mass, union_bits, step_bits, eta, rows, nq);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

template <int F>
static cudaError_t launch_pooled(const float* mass, uint32_t* union_bits, uint32_t* step_bits,
                                 float eta, int BH, int nq, cudaStream_t stream) {
  const int nQ = nq / F;
  const long long crows = (long long)BH * nQ;
  const int Wc = (nQ + 31) / 32;
  const int warps_per_block = 8;
  const unsigned grid = (unsigned)((crows + warps_per_block - 1) / warps_per_block);
  const dim3 block(32 * warps_per_block);
  if (Wc <= 1)
    select_union_pooled_kernel<1, F><<<grid, block, 0, stream>>>(mass, union_bits, step_bits, eta,
                                                                 crows, nq);
  else if (Wc <= 2)
    select_union_pooled_kernel<2, F><<<grid, block, 0, stream>>>(mass, union_bits, step_bits, eta,
                                                                 crows, nq);
  else if (Wc <= 4)
    select_union_pooled_kernel<4, F><<<grid, block, 0, stream>>>(mass, union_bits, step_bits, eta,
                                                                 crows, nq);
  else if (Wc <= 8)
    select_union_pooled_kernel<8, F><<<grid, block, 0, stream>>>(mass, union_bits, step_bits, eta,
                                                                 crows, nq);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_select_union_blocks(const float* mass, uint32_t* union_bits,
                                       uint32_t* step_bits, float eta, int factor, int BH, int nq,
                                       cudaStream_t stream) {
  if (factor == 1)
    return launch_select_union(mass, union_bits, step_bits, eta, BH, nq, stream);
  if (nq % factor != 0) return cudaErrorInvalidValue;
  if (factor == 2) return launch_pooled<2>(mass, union_bits, step_bits, eta, BH, nq, stream);
  if (factor == 4) return launch_pooled<4>(mass, union_bits, step_bits, eta, BH, nq, stream);
  return cudaErrorInvalidValue;
}

// ----------------------------------------------------------------------------------------
// Selection-only controls and the retained-mass metric (WISE paper appendix B,
// "Intervention controls" and "Evaluation metrics").  One warp per (bh, q) row, the same
// lane/slot layout as above: lane l holds blocks l, l + 32, ...

template <int MAXW>
__device__ __forceinline__ void load_mass_row(const float* __restrict__ mrow, int q, int W,
                                              int lane, float (&v)[MAXW], bool (&ok)[MAXW]) {
#pragma unroll
  for (int s = 0; s < MAXW; ++s) {
    const int kb = s * 32 + lane;
    ok[s] = (s < W) && (kb <= q);
    v[s] = ok[s] ? mrow[kb] : 0.f;
  }
}

// in[s] = bit (s * 32 + lane) of a [W]-word mask row, admissible blocks only.
template <int MAXW>
__device__ __forceinline__ void load_bits_row(const uint32_t* __restrict__ brow,
                                              const bool (&ok)[MAXW], int lane,
                                              bool (&in)[MAXW]) {
#pragma unroll
  for (int s = 0; s < MAXW; ++s) in[s] = ok[s] && ((brow[s] >> lane) & 1u);
}

template <int MAXW>
__device__ __forceinline__ int warp_count_ge(const float (&v)[MAXW], const bool (&ok)[MAXW],
                                             float tau) {
  int c = 0;
#pragma unroll
  for (int s = 0; s < MAXW; ++s) c += __popc(__ballot_sync(0xffffffffu, ok[s] && v[s] >= tau));
  return c;
}

// TopK with ties to the lower index: tau = the largest float with #{v >= tau} >= K, by
// bisection over the bit patterns (v >= 0); keep v > tau, then blocks equal to tau in
// ascending index order until K are kept.
template <int MAXW>
__device__ __forceinline__ void topk_cut(const float (&v)[MAXW], const bool (&ok)[MAXW], int K,
                                         int lane, bool (&sel)[MAXW]) {
  uint32_t lo = 0u, hi = 0x7F800000u;  // count(lo) >= K (every admissible block), count(hi) < K
  while (hi - lo > 1u) {
    const uint32_t mid = lo + ((hi - lo) >> 1);
    if (warp_count_ge<MAXW>(v, ok, __uint_as_float(mid)) >= K)
      lo = mid;
    else
      hi = mid;
  }
  const float tau = __uint_as_float(lo);
  int kept = warp_count_ge<MAXW>(v, ok, __uint_as_float(hi));  // strictly above tau
#pragma unroll
  for (int s = 0; s < MAXW; ++s) sel[s] = ok[s] && v[s] > tau;
#pragma unroll
  for (int s = 0; s < MAXW; ++s) {
    uint32_t ties = __ballot_sync(0xffffffffu, ok[s] && v[s] == tau);
    while (ties != 0u && kept < K) {
      const int b = __ffs(ties) - 1;
      ties &= ties - 1u;
      ++kept;
      if (lane == b) sel[s] = true;
    }
  }
}

template <int MAXW>
__device__ __forceinline__ void store_bits_row(uint32_t* __restrict__ dst, int W, int lane,
                                               const bool (&sel)[MAXW]) {
  uint32_t word = 0u;
#pragma unroll
  for (int s = 0; s < MAXW; ++s) {
    const uint32_t w = __ballot_sync(0xffffffffu, sel[s]);
    if (lane == s) word = w;
  }
  if (lane < W) dst[lane] = word;
}

// kSize: SizeMatched, K_q = |W_q| blocks of largest mass.  kMass: MassMatched, the
// cumulative-eta cut at eta = m_q, the mass of W_q, in the cut's own fixed-point units
// (so a ranking prefix holding W_q's blocks reaches m_q exactly).
enum ControlKind { kSizeMatched = 0, kMassMatched = 1 };

template <int MAXW, int KIND>
__global__ void __launch_bounds__(256)
    select_control_kernel(const float* __restrict__ mass, const uint32_t* __restrict__ ref,
                          uint32_t* __restrict__ out, long long rows, int nq) {
  __shared__ __align__(16) uint32_t hist_s[8][256];   // cut_at's digit histogram, per warp
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;  // warp-uniform
  const int W = (nq + 31) >> 5;
  const int q = (int)(row % nq);
  float v[MAXW];
  bool ok[MAXW], in[MAXW], sel[MAXW];
  load_mass_row<MAXW>(mass + row * (long long)nq, q, W, lane, v, ok);
  load_bits_row<MAXW>(ref + row * W, ok, lane, in);
  if (KIND == kSizeMatched) {
    int K = 0;
#pragma unroll
    for (int s = 0; s < MAXW; ++s) K += __popc(__ballot_sync(0xffffffffu, in[s]));
    if (K == 0) {
#pragma unroll
      for (int s = 0; s < MAXW; ++s) sel[s] = false;
    } else {
      topk_cut<MAXW>(v, ok, K, lane, sel);
    }
  } else {
    // m_q in the cut's units: the sum of the reference blocks' units, so a ranking
    // prefix holding exactly W_q's blocks reaches it exactly
    uint32_t part = 0u;
#pragma unroll
    for (int s = 0; s < MAXW; ++s) part += in[s] ? cut_units(v[s]) : 0u;
    const uint32_t m = __reduce_add_sync(0xffffffffu, part);
    if (m == 0u) {
#pragma unroll
      for (int s = 0; s < MAXW; ++s) sel[s] = false;
    } else if (m >= (uint32_t)kCutScale) {   // m_q >= 1 keeps every admissible block
#pragma unroll
      for (int s = 0; s < MAXW; ++s) sel[s] = ok[s];
    } else {
      cut_at<MAXW>(v, ok, m, lane, sel, hist_s[threadIdx.x >> 5]);
    }
  }
  store_bits_row<MAXW>(out + row * W, W, lane, sel);
}

// retained[row] = sum of mass[row][b] over set bits b <= q (fp32: per lane, then a
// butterfly over the lanes).
template <int MAXW>
__global__ void __launch_bounds__(256)
    support_mass_kernel(const float* __restrict__ mass, const uint32_t* __restrict__ bits,
                        float* __restrict__ retained, long long rows, int nq) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;  // warp-uniform
  const int W = (nq + 31) >> 5;
  const int q = (int)(row % nq);
  float v[MAXW];
  bool ok[MAXW], in[MAXW];
  load_mass_row<MAXW>(mass + row * (long long)nq, q, W, lane, v, ok);
  load_bits_row<MAXW>(bits + row * W, ok, lane, in);
  float a = 0.f;
#pragma unroll
  for (int s = 0; s < MAXW; ++s) a += in[s] ? v[s] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
  if (lane == 0) retained[row] = a;
}

// Calls f(std::integral_constant<int, MAXW>) for the smallest MAXW in {1, 2, 4, 8, 16} >= W.
template <typename Fn>
static cudaError_t by_width(int W, Fn&& f) {
  if (W <= 1)
    f(std::integral_constant<int, 1>{});
  else if (W <= 2)
    f(std::integral_constant<int, 2>{});
  else if (W <= 4)
    f(std::integral_constant<int, 4>{});
  else if (W <= 8)
    f(std::integral_constant<int, 8>{});
  else if (W <= 16)
    f(std::integral_constant<int, 16>{});
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_select_control(const float* mass, const uint32_t* ref_bits, uint32_t* out_bits,
                                  int kind, int BH, int nq, cudaStream_t stream) {
  const long long rows = (long long)BH * nq;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  return by_width((nq + 31) / 32, [&](auto w) {
    constexpr int M = decltype(w)::value;
    if (kind == kSizeMatched)
      select_control_kernel<M, kSizeMatched><<<grid, 256, 0, stream>>>(mass, ref_bits, out_bits,
                                                                       rows, nq);
    else
      select_control_kernel<M, kMassMatched><<<grid, 256, 0, stream>>>(mass, ref_bits, out_bits,
                                                                       rows, nq);
  });
}

cudaError_t launch_support_mass(const float* mass, const uint32_t* bits, float* retained, int BH,
                                int nq, cudaStream_t stream) {
  const long long rows = (long long)BH * nq;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  return by_width((nq + 31) / 32, [&](auto w) {
    constexpr int M = decltype(w)::value;
    support_mass_kernel<M><<<grid, 256, 0, stream>>>(mass, bits, retained, rows, nq);
  });
}

}  // namespace wise
