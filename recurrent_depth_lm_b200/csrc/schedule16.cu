// schedule16.cu -- the CSR schedule of a 16-token working set, run on 32 x 32 tiles.
//
// Wan & Chen, "Attention Routing Stabilizes Early: Working-Set Inference for
// Recurrent-Depth Language Models", appendix C.6 ("Block-Size Tradeoff") evaluates
// B = 16 next to B = 32; appendix B ("Sparse-kernel implementation") defines the
// schedule as row offsets plus active key blocks per query block.  Here the
// attention tiles stay 32 x 32: the schedule lists a 32-token key block for a
// 32-token query block when any of its four 16 x 16 sub-blocks is in the working
// set, and each entry carries those four bits (bit 2a + c: 16-row 2q + a keeps
// 16-block 2b + c), so the kernel masks exactly the 16-token support.
//
//   fold : union16 [BH, 2nq, W16] -> bits32 [BH, nq, W] (thread per output word)
//   (the 32-token schedule builder runs on bits32)
//   sub  : one warp per 32-row, lanes over its entries, four bit reads each

#include <cstdint>

#include "wise_internal.h"

namespace wise {

// Bits 0, 2, 4, ... of x packed into bits 0, 1, 2, ... (a 64 -> 32 bit unshuffle).
__device__ __forceinline__ uint32_t even_bits(uint64_t x) {
  x &= 0x5555555555555555ull;
  x = (x | (x >> 1)) & 0x3333333333333333ull;
  x = (x | (x >> 2)) & 0x0F0F0F0F0F0F0F0Full;
  x = (x | (x >> 4)) & 0x00FF00FF00FF00FFull;
  x = (x | (x >> 8)) & 0x0000FFFF0000FFFFull;
  x = (x | (x >> 16)) & 0x00000000FFFFFFFFull;
  return (uint32_t)x;
}

__global__ void __launch_bounds__(256)
    fold16_kernel(const uint32_t* __restrict__ u16, uint32_t* __restrict__ b32, long long items,
                  int nq) {
  const long long it = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (it >= items) return;
  const int W = (nq + 31) >> 5;
  const int n16 = 2 * nq;
  const int W16 = (n16 + 31) >> 5;
  const long long row = it / W;  // (bh, q)
  const int w = (int)(it % W);
  const long long bh = row / nq;
  const int q = (int)(row % nq);
  uint32_t out = 0u;
#pragma unroll
  for (int a = 0; a < 2; ++a) {
    const int r16 = 2 * q + a;
    const uint32_t* src = u16 + (bh * n16 + r16) * W16;
    // 16-blocks 64 w .. 64 w + 63 are words 2 w and 2 w + 1 of the 16-row
    const uint64_t lo = (2 * w < W16) ? src[2 * w] : 0u;
    const uint64_t hi = (2 * w + 1 < W16) ? src[2 * w + 1] : 0u;
    uint64_t x = lo | (hi << 32);
    const int keep = r16 - 64 * w;  // causal: 16-block <= r16
    if (keep < 0)
      x = 0ull;
    else if (keep < 63)
      x &= (2ull << keep) - 1ull;
    out |= even_bits(x | (x >> 1));
  }
  b32[it] = out;
}

__global__ void __launch_bounds__(256)
    sub16_kernel(const uint32_t* __restrict__ u16, const int32_t* __restrict__ row_offsets,
                 const int32_t* __restrict__ col_idx, uint8_t* __restrict__ sub, long long cap,
                 long long rows, int nq) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;  // warp-uniform
  const int n16 = 2 * nq;
  const int W16 = (n16 + 31) >> 5;
  const long long bh = row / nq;
  const int q = (int)(row % nq);
  const long long beg = row_offsets[row];
  long long end = row_offsets[row + 1];
  if (end > cap) end = cap;
  for (long long e = beg + lane; e < end; e += 32) {
    const int b = col_idx[e];
    uint32_t bits = 0u;
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const int r16 = 2 * q + a;
      const uint32_t* src = u16 + (bh * n16 + r16) * W16;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int b16 = 2 * b + c;
        if (b16 <= r16 && ((src[b16 >> 5] >> (b16 & 31)) & 1u)) bits |= 1u << (2 * a + c);
      }
    }
    sub[e] = (uint8_t)bits;
  }
}

cudaError_t launch_fold16(const uint32_t* union16, uint32_t* bits32, int BH, int nq,
                          cudaStream_t stream) {
  const long long items = (long long)BH * nq * ((nq + 31) / 32);
  const unsigned grid = (unsigned)((items + 255) / 256);
  fold16_kernel<<<grid, 256, 0, stream>>>(union16, bits32, items, nq);
  return cudaGetLastError();
}

cudaError_t launch_sub16(const uint32_t* union16, const int32_t* row_offsets,
                         const int32_t* col_idx, uint8_t* sub, long long capacity, int BH,
                         int nq, cudaStream_t stream) {
  const long long rows = (long long)BH * nq;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  sub16_kernel<<<grid, 256, 0, stream>>>(union16, row_offsets, col_idx, sub, capacity, rows, nq);
  return cudaGetLastError();
}

}  // namespace wise
