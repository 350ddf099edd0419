// schedule.cu -- compaction of the working-set bitmask into the CSR schedule.
//
// Wan & Chen, "Attention Routing Stabilizes Early: Working-Set Inference for
// Recurrent-Depth Language Models", appendix B ("Sparse-kernel
// implementation"): for each recurrent block, head and query block the active
// key blocks are a reusable GPU-resident CSR schedule (row offsets + active
// block indices), built once after discovery.
//
// Three launches over blocks of kSchedThreads rows (bh, q):
//   count : popcount of each row's admissible bits (thread per row), block sums
//           -> workspace
//   scan  : exclusive scan of the block sums (one CTA), total -> row_offsets[rows]
//   emit  : the block's bitmask words are staged in shared memory; block-local
//           exclusive scan + block base -> row_offsets[row]; then every
//           (row, word) item is expanded by its own thread at the row's offset
//           plus the popcount of the row's earlier words (ascending order,
//           clamped to capacity).

#include <cstdint>

#include "wise_internal.h"

namespace wise {

constexpr int kSchedThreads = 256;
constexpr int kSchedWarps = kSchedThreads / 32;
constexpr int kMaxSchedWords = 16;   // bitmask words per row: nq <= 512

__device__ __forceinline__ uint32_t admissible_word(const uint32_t* ub, long long row, int W, int w,
                                                    int q) {
  const int base = w * 32;
  if (base > q) return 0u;
  uint32_t word = ub[row * W + w];
  const int hi = q - base;  // keep bits 0..hi
  if (hi < 31) word &= (2u << hi) - 1u;
  return word;
}

__device__ __forceinline__ int row_count(const uint32_t* ub, long long row, int W, int nq) {
  const int q = (int)(row % nq);
  int c = 0;
  for (int w = 0; w < W; ++w) c += __popc(admissible_word(ub, row, W, w, q));
  return c;
}

// Inclusive scan over the block's kSchedThreads threads; returns the inclusive value, *total = block sum.
__device__ __forceinline__ int block_inclusive_scan(int x, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < kSchedWarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < kSchedWarps) warp_sums[lane] = s;
  }
  __syncthreads();
  if (warp > 0) x += warp_sums[warp - 1];
  *total = warp_sums[kSchedWarps - 1];
  return x;
}

__global__ void __launch_bounds__(kSchedThreads)
    sched_count_kernel(const uint32_t* __restrict__ ub, int* __restrict__ block_sums, long long rows,
                       int nq) {
  __shared__ int warp_sums[32];
  const int W = (nq + 31) >> 5;
  const long long row = (long long)blockIdx.x * kSchedThreads + threadIdx.x;
  const int c = row < rows ? row_count(ub, row, W, nq) : 0;
  int total;
  block_inclusive_scan(c, warp_sums, &total);
  if (threadIdx.x == 0) block_sums[blockIdx.x] = total;
}

// Exclusive scan of nblocks block sums in place; writes the grand total to *total_out.
__global__ void __launch_bounds__(kSchedThreads)
    sched_scan_kernel(int* __restrict__ block_sums, int nblocks, int32_t* __restrict__ total_out) {
  __shared__ int warp_sums[32];
  int carry = 0;
  for (int base = 0; base < nblocks; base += kSchedThreads) {
    const int idx = base + threadIdx.x;
    const int x = idx < nblocks ? block_sums[idx] : 0;
    int tot;
    const int inc = block_inclusive_scan(x, warp_sums, &tot);
    if (idx < nblocks) block_sums[idx] = carry + inc - x;
    carry += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) *total_out = carry;
}

__global__ void __launch_bounds__(kSchedThreads)
    sched_emit_kernel(const uint32_t* __restrict__ ub, const int* __restrict__ block_base,
                      int32_t* __restrict__ row_offsets, int32_t* __restrict__ col_idx,
                      long long capacity, long long rows, int nq) {
  __shared__ int warp_sums[32];
  __shared__ int row_off[kSchedThreads];
  __shared__ uint32_t words[kSchedThreads * kMaxSchedWords];
  const int W = (nq + 31) >> 5;
  const long long row0 = (long long)blockIdx.x * kSchedThreads;
  const int nrows = (rows - row0 < kSchedThreads) ? (int)(rows - row0) : kSchedThreads;
  // stage this block's admissible bitmask words (coalesced)
  for (int x = threadIdx.x; x < nrows * W; x += kSchedThreads) {
    const int rr = x / W, w = x % W;
    const long long r = row0 + rr;
    words[rr * W + w] = admissible_word(ub, r, W, w, (int)(r % nq));
  }
  __syncthreads();
  int c = 0;
  if (threadIdx.x < nrows)
    for (int w = 0; w < W; ++w) c += __popc(words[threadIdx.x * W + w]);
  int total;
  const int inc = block_inclusive_scan(c, warp_sums, &total);
  const int off = block_base[blockIdx.x] + inc - c;
  row_off[threadIdx.x] = off;
  if (threadIdx.x < nrows) row_offsets[row0 + threadIdx.x] = off;
  __syncthreads();
  // expand every (row, word) item independently: its bits go after the row's earlier words
  for (int x = threadIdx.x; x < nrows * W; x += kSchedThreads) {
    const int rr = x / W, w = x % W;
    uint32_t word = words[rr * W + w];
    long long at = row_off[rr];
    for (int w2 = 0; w2 < w; ++w2) at += __popc(words[rr * W + w2]);
    while (word != 0u) {
      const int b = __ffs(word) - 1;
      word &= word - 1u;
      if (at < capacity) col_idx[at] = w * 32 + b;
      ++at;
    }
  }
}

size_t schedule_workspace_bytes(long long rows) {
  const long long nblocks = (rows + kSchedThreads - 1) / kSchedThreads;
  return (size_t)(nblocks < 1 ? 1 : nblocks) * sizeof(int);
}

cudaError_t launch_build_schedule(const uint32_t* union_bits, int32_t* row_offsets,
                                  int32_t* col_idx, long long capacity, void* workspace,
                                  long long rows, int nq, cudaStream_t stream) {
  const int nblocks = (int)((rows + kSchedThreads - 1) / kSchedThreads);
  int* block_sums = static_cast<int*>(workspace);
  sched_count_kernel<<<nblocks, kSchedThreads, 0, stream>>>(union_bits, block_sums, rows, nq);
  sched_scan_kernel<<<1, kSchedThreads, 0, stream>>>(block_sums, nblocks, row_offsets + rows);
  sched_emit_kernel<<<nblocks, kSchedThreads, 0, stream>>>(union_bits, block_sums, row_offsets,
                                                           col_idx, capacity, rows, nq);
  return cudaGetLastError();
}

}  // namespace wise
