// attn.cu -- tcgen05/TMEM attention kernels of the WISE hot path (sm_100a).
//
// One persistent, warp-specialised kernel template covers three modes:
//   kDense  : exploration-step causal attention (all admissible key blocks),
//   kSparse : late-step attention over a CSR key-block schedule,
//   kMass   : the block-mass pass of an exploration window step.
//
// Semantics follow Wan & Chen, "Attention Routing Stabilizes Early:
// Working-Set Inference for Recurrent-Depth Language Models": section 3
// (A = softmax(QK^T/sqrt(d_h) + M), O = AV), section 5.1 (block mass
// r_qb = mean over query rows of block q of the row's mass in key block b),
// section 5.2 (reuse mask: keys outside the working set are excluded) and
// section 7.4 (absent blocks are skipped; scoring, causal mask, online
// softmax and value aggregation are fused).
//
// Tiling.  A CTA tile is 128 query rows = 4 query blocks of 32 (one TMEM lane
// slice of 32 rows per softmax warp, i.e. one query block per warp).  Each
// iteration gathers up to 4 key blocks (128 keys) with one 32-row TMA box per
// block and panel, so the tile's key list may be any ascending set of blocks.
// A slot's "owner mask" says which of the tile's 4 query blocks may see it;
// rows of other query blocks get probability 0 for it.
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = TMEM allocator +
// single-thread MMA issuer, warps 2..5 = softmax / epilogue (one row each).
//
// Shared memory (128-byte swizzle, 1024-byte aligned panels of 64 columns):
//   Q tile [128 x d], NS stages of K (and V) [128 keys x d], P [128 x 128] bf16.
// Tensor memory: S double buffer (2 x 128 fp32 columns) + O (d columns).

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100.cuh"
#include "wise_internal.h"

namespace wise {

constexpr int kBM = 128;        // query rows per tile
constexpr int kSlots = 4;       // key blocks per iteration
constexpr int kThreads = 192;
constexpr int kPanelRowBytes = 128;            // 64 bf16 per swizzled row
constexpr int kPanelBytes = kBM * kPanelRowBytes;  // one 128-row panel = 16 KB
constexpr int kMaxWords = 16;   // schedule bitmask words per query block (nq <= 512)

template <int D, int MODE>
struct Cfg {
  static constexpr int kPanels = (D + 63) / 64;
  static constexpr bool kAttn = MODE != kModeMass;
  static constexpr int kStages = (D <= 64) ? 4 : (kAttn ? 2 : 4);
  static constexpr int kTileBytes = kPanels * kPanelBytes;  // Q tile, K stage, V stage
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffP = kOffV + (kAttn ? kStages * kTileBytes : 0);
  static constexpr int kOffInfo = kOffP + (kAttn ? 2 * kPanelBytes : 0);
  static constexpr int kInfoInts = 16;
  static constexpr int kOffMask = kOffInfo + kStages * kInfoInts * 4;
  static constexpr int kOffBar = kOffMask + 4 * kMaxWords * 4;
  // barriers: q_full, q_empty, kv_full[S], kv_empty[S], s_full[2], s_free[2], p_full, o_done,
  // o_staged, final
  static constexpr int kNumBars = 2 + 2 * kStages + 4 + 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = kAttn ? 512 : 256;
  static constexpr uint32_t kOCol = 256;
};

struct StageInfo {
  int nslots;
  int last;
  int kb[kSlots];
  int own[kSlots];
};

// ---------------------------------------------------------------- key-block lists

// Dense causal list for tile (q-blocks 4*Qt .. 4*Qt+3): every kb <= last q-block,
// owner bits r with kb <= 4*Qt + r < nq.
struct DenseList {
  int next, end, qb0, nq;
  __device__ void init(int Qt, int nq_) {
    nq = nq_;
    qb0 = Qt * 4;
    next = 0;
    end = min(qb0 + 3, nq - 1) + 1;
  }
  __device__ bool pop(int& kb, int& own) {
    if (next >= end) return false;
    kb = next++;
    own = 0;
#pragma unroll
    for (int r = 0; r < 4; ++r)
      if (qb0 + r < nq && kb <= qb0 + r) own |= 1 << r;
    return true;
  }
};

// Sparse list: the union of the tile's 4 CSR rows, as per-row bitmasks built in
// shared memory by the producer warp; popped in ascending block order.
struct MaskList {
  const uint32_t* mask;  // [4][kMaxWords]
  int words, w;
  uint32_t cur;
  __device__ void init(const uint32_t* m, int words_) {
    mask = m;
    words = words_;
    w = 0;
    cur = words > 0 ? (m[0] | m[kMaxWords] | m[2 * kMaxWords] | m[3 * kMaxWords]) : 0u;
  }
  __device__ bool pop(int& kb, int& own) {
    while (cur == 0) {
      if (++w >= words) return false;
      cur = mask[w] | mask[kMaxWords + w] | mask[2 * kMaxWords + w] | mask[3 * kMaxWords + w];
    }
    int bit = __ffs(cur) - 1;
    cur &= cur - 1;
    kb = w * 32 + bit;
    own = 0;
#pragma unroll
    for (int r = 0; r < 4; ++r)
      if ((mask[r * kMaxWords + w] >> bit) & 1u) own |= 1 << r;
    return true;
  }
};

// Build the 4 per-row bitmasks of a sparse tile (whole producer warp).
__device__ void build_tile_masks(uint32_t* mask, const AttnParams& p, int bh, int Qt, int lane) {
  const int words = (p.nq + 31) / 32;
  for (int x = lane; x < 4 * kMaxWords; x += 32) mask[x] = 0u;
  __syncwarp();
  for (int r = 0; r < 4; ++r) {
    const int qb = Qt * 4 + r;
    if (qb >= p.nq) break;
    const long long row = (long long)bh * p.nq + qb;
    long long beg = p.row_offsets[row];
    long long end = p.row_offsets[row + 1];
    bool bad = false;
    if (beg < 0 || end > p.col_count || beg > end) {
      bad = true;
      beg = end = 0;
    }
    for (long long e = beg + lane; e < end; e += 32) {
      const int kb = p.col_idx[e];
      if (kb >= 0 && kb <= qb && kb < words * 32)
        atomicOr(&mask[r * kMaxWords + (kb >> 5)], 1u << (kb & 31));
      else
        bad = true;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.status, kStatusBadSchedule);
  }
  __syncwarp();
}

// ---------------------------------------------------------------- helpers

__device__ __forceinline__ void reg_fence32(uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]));
}

// Warp-uniform bounded wait: every lane polls, the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          unsigned int* status) {
  bool ok = mbar_wait(bar, parity, abort, status);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) *abort = 1;
  return ok;
}

__device__ __forceinline__ void decode_tile(int tile, int BH, int ntq, int& bh, int& Qt) {
  // heaviest tiles (largest Qt, most key blocks) first
  Qt = ntq - 1 - tile / BH;
  bh = tile % BH;
}

// ---------------------------------------------------------------- the kernel

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                const AttnParams p) {
  using C = Cfg<D, MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t sQ = smem_u32(smem + C::kOffQ);
  const uint32_t sK = smem_u32(smem + C::kOffK);
  const uint32_t sV = smem_u32(smem + C::kOffV);
  const uint32_t sP = smem_u32(smem + C::kOffP);
  StageInfo* info = (StageInfo*)(smem + C::kOffInfo);
  uint32_t* tile_mask = (uint32_t*)(smem + C::kOffMask);
  const uint32_t bar0 = smem_u32(smem + C::kOffBar);
  const uint32_t bar_q_full = bar0;
  const uint32_t bar_q_empty = bar0 + 8;
  auto bar_kv_full = [&](int s) { return bar0 + 16 + 8 * s; };
  auto bar_kv_empty = [&](int s) { return bar0 + 16 + 8 * C::kStages + 8 * s; };
  const uint32_t barS = bar0 + 16 + 16 * C::kStages;
  auto bar_s_full = [&](int b) { return barS + 8 * b; };
  auto bar_s_free = [&](int b) { return barS + 16 + 8 * b; };
  const uint32_t bar_p_full = barS + 32;
  const uint32_t bar_o_done = barS + 40;
  const uint32_t bar_o_staged = barS + 48;
  const uint32_t bar_final = barS + 56;
  volatile int* abort_flag = (volatile int*)(smem + C::kOffMisc);
  uint32_t* tmem_slot = (uint32_t*)(smem + C::kOffMisc + 4);

  const int ntq = (p.nq + 3) / 4;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar_kv_full(s), 1);
      // mass mode: freed by the QK commit AND by every softmax thread once it has
      // read the stage's slot info (128 + 1 arrivals); attention mode: by the PV commit.
      mbar_init(bar_kv_empty(s), C::kAttn ? 1 : 129);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_s_full(b), 1);
      mbar_init(bar_s_free(b), 128);
    }
    mbar_init(bar_p_full, 128);
    mbar_init(bar_o_done, 1);
    mbar_init(bar_o_staged, 128);
    mbar_init(bar_final, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ======================================================= producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      if (C::kAttn) {
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmO);
      }
    }
    uint32_t it = 0;
    int tl = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tl) {
      int bh, Qt;
      decode_tile(tile, p.BH, ntq, bh, Qt);
      if (MODE == kModeSparse) {
        // The previous tile's list has been fully issued (only lane 0 reads it).
        build_tile_masks(tile_mask, p, bh, Qt, lane);
      }
      if (lane == 0) {
        if (tl > 0 && !mbar_wait(bar_q_empty, (tl - 1) & 1, abort_flag, p.status)) ok = false;
        if (ok) {
          mbar_arrive_expect_tx(bar_q_full, C::kTileBytes);
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_3d(sQ + pn * kPanelBytes, &tmQ, bar_q_full, pn * 64, Qt * kBM, bh);
        }
        DenseList dl;
        MaskList ml;
        if (MODE == kModeSparse)
          ml.init(tile_mask, (p.nq + 31) / 32);
        else
          dl.init(Qt, p.nq);
        bool first = true;
        while (ok) {
          const int stage = it % C::kStages;
          if (it >= (uint32_t)C::kStages &&
              !mbar_wait(bar_kv_empty(stage), ((it / C::kStages) - 1) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          StageInfo& si = info[stage];
          int n = 0;
          int kb, own;
          while (n < kSlots && (MODE == kModeSparse ? ml.pop(kb, own) : dl.pop(kb, own))) {
            si.kb[n] = kb;
            si.own[n] = own;
            ++n;
          }
          if (n == 0 && first) {  // empty tile: one fully masked slot keeps the pipeline uniform
            si.kb[0] = 0;
            si.own[0] = 0;
            n = 1;
          }
          bool last;
          if (n < kSlots) {
            last = true;
          } else {
            // peek: is anything left?
            if (MODE == kModeSparse) {
              MaskList t = ml;
              last = !t.pop(kb, own);
            } else {
              last = dl.next >= dl.end;
            }
          }
          if (n == 0) break;  // cannot happen (handled above) but keeps the loop finite
          si.nslots = n;
          si.last = last ? 1 : 0;
          const uint32_t bytes = (uint32_t)n * 32 * kPanelRowBytes * C::kPanels * (C::kAttn ? 2 : 1);
          mbar_arrive_expect_tx(bar_kv_full(stage), bytes);
          const uint32_t kbase = sK + stage * C::kTileBytes;
          const uint32_t vbase = sV + stage * C::kTileBytes;
          for (int s = 0; s < n; ++s) {
            for (int pn = 0; pn < C::kPanels; ++pn) {
              tma_load_3d(kbase + pn * kPanelBytes + s * 32 * kPanelRowBytes, &tmK,
                          bar_kv_full(stage), pn * 64, si.kb[s] * 32, bh);
              if (C::kAttn)
                tma_load_3d(vbase + pn * kPanelBytes + s * 32 * kPanelRowBytes, &tmV,
                            bar_kv_full(stage), pn * 64, si.kb[s] * 32, bh);
            }
          }
          ++it;
          first = false;
          if (last) break;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      it = __shfl_sync(0xffffffffu, it, 0);
    }
    // Drain: let the last issued loads land before the CTA can exit.
    if (lane == 0) {
      const uint32_t from = it > (uint32_t)C::kStages ? it - C::kStages : 0u;
      for (uint32_t j = from; j < it; ++j) {
        volatile int dummy = 0;
        mbar_wait(bar_kv_full(j % C::kStages), (j / C::kStages) & 1, &dummy, p.status);
      }
    }
  } else if (warp == 1) {
    // ======================================================= MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);
      uint32_t it = 0;
      int tl = 0;
      bool ok = true;
      bool issued = false;
      // Issues S_j = Q K_j^T; returns the stage's slot count and last flag, read
      // before the stage can be released.
      auto issue_qk = [&](uint32_t j, int& ns, int& last) -> bool {
        const int stage = j % C::kStages;
        if (!mbar_wait(bar_kv_full(stage), (j / C::kStages) & 1, abort_flag, p.status)) return false;
        if (j >= 2 && !mbar_wait(bar_s_free(j & 1), ((j >> 1) - 1) & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        ns = info[stage].nslots;
        last = info[stage].last;
        const uint32_t idesc = idesc_bf16_f32(128, 32 * ns, 0, 0);
        const uint32_t d_tmem = tmem_base + (j & 1) * 128;
        const uint32_t kbase = sK + stage * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kPanelBytes + (kk & 3) * 32;
          mma_bf16_ss(d_tmem, smem_desc_sw128(sQ + off, 16, 1024),
                      smem_desc_sw128(kbase + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_s_full(j & 1));
        if (!C::kAttn) mma_commit(bar_kv_empty(stage));
        issued = true;
        return true;
      };
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tl) {
        if (!mbar_wait(bar_q_full, tl & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t g0 = it;
        int ns = 0, last = 1;
        if (!issue_qk(it, ns, last)) {
          ok = false;
          break;
        }
        while (true) {
          const int stage = it % C::kStages;
          int ns_next = 0, last_next = 1;
          if (!last && !issue_qk(it + 1, ns_next, last_next)) {
            ok = false;
            break;
          }
          if (C::kAttn) {
            if (!mbar_wait(bar_p_full, it & 1, abort_flag, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t vbase = sV + stage * C::kTileBytes;
            for (int kk = 0; kk < 2 * ns; ++kk) {
              const uint64_t a = smem_desc_sw128(sP + (kk >> 2) * kPanelBytes + (kk & 3) * 32, 16, 1024);
              const uint64_t b = smem_desc_sw128(vbase + kk * 16 * kPanelRowBytes, kPanelBytes, 1024);
              mma_bf16_ss(tmem_base + C::kOCol, a, b, idesc_o, (it > g0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(bar_o_done);
            mma_commit(bar_kv_empty(stage));
          }
          ++it;
          if (last) break;
          ns = ns_next;
          last = last_next;
        }
        if (!ok) break;
        if (!C::kAttn) mma_commit(bar_q_empty);  // Q is free once this tile's QK MMAs finish
      }
      if (issued) {
        mma_commit(bar_final);
        volatile int dummy = 0;
        mbar_wait(bar_final, 0, &dummy, p.status);
      }
    }
    __syncwarp();
  } else {
    // ======================================================= softmax / epilogue
    const int wg = warp & 3;         // TMEM lane quarter owned by this warp
    const int r = wg * 32 + lane;    // row within the tile
    const uint32_t t_row = tmem_base + ((uint32_t)(wg * 32) << 16);
    const float sl2 = p.scale_log2;
    uint32_t it = 0;
    int tl = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tl) {
      int bh, Qt;
      decode_tile(tile, p.BH, ntq, bh, Qt);
      const int qb = Qt * 4 + wg;      // this warp's query block
      const int i = qb * 32 + lane;    // query row within the head
      float m = -INFINITY, l = 0.f;
      float lse_l2 = 0.f;
      if (!C::kAttn && i < p.n) lse_l2 = p.lse_in[(long long)bh * p.n + i] * 1.4426950408889634f;
      const uint32_t g0 = it;
      while (true) {
        const int stage = it % C::kStages;
        if (!warp_wait(bar_kv_full(stage), (it / C::kStages) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        const int ns = info[stage].nslots;
        const int last = info[stage].last;
        int kbs[kSlots], vld[kSlots];
#pragma unroll
        for (int s = 0; s < kSlots; ++s) {
          kbs[s] = info[stage].kb[s];
          vld[s] = (s < ns) && ((info[stage].own[s] >> wg) & 1);
        }
        if (!C::kAttn) mbar_arrive(bar_kv_empty(stage));  // slot info consumed
        if (!warp_wait(bar_s_full(it & 1), (it >> 1) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[kSlots][32];
#pragma unroll
        for (int s = 0; s < kSlots; ++s)
          if (vld[s]) tmem_ld32(t_row + (it & 1) * 128 + s * 32, sr[s]);
        tmem_wait_ld();
#pragma unroll
        for (int s = 0; s < kSlots; ++s) reg_fence32(sr[s]);
        tc_fence_before();
        mbar_arrive(bar_s_free(it & 1));

        if (!C::kAttn) {
          // ---------------- block mass: sum_j exp(s_ij*scale - lse_i) over the block, mean over rows
#pragma unroll
          for (int s = 0; s < kSlots; ++s) {
            if (!vld[s]) continue;
            const bool diag = kbs[s] == qb;
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float x = __uint_as_float(sr[s][c]);
              const float e = fast_exp2(fmaf(x, sl2, -lse_l2));
              acc += (diag && c > lane) ? 0.f : e;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0)
              p.mass[((long long)bh * p.nq + qb) * p.nq + kbs[s]] = acc * (1.0f / 32.0f);
          }
        } else {
          // ---------------- online softmax (log2 domain, lazily rescaled)
          float mx = -INFINITY;
#pragma unroll
          for (int s = 0; s < kSlots; ++s) {
            const bool diag = kbs[s] == qb;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              float x = vld[s] ? __uint_as_float(sr[s][c]) * sl2 : -INFINITY;
              if (diag && c > lane) x = -INFINITY;
              sr[s][c] = __float_as_uint(x);
              mx = fmaxf(mx, x);
            }
          }
          const float m_new = fmaxf(m, mx);
          const bool need = m_new > m + 8.0f;   // true on the first finite score
          const bool warp_need = __any_sync(0xffffffffu, need);
          const float m_use = warp_need ? m_new : m;
          const float alpha = (warp_need && m != -INFINITY) ? fast_exp2(m - m_use) : 1.0f;
          float rs = 0.f;
#pragma unroll
          for (int s = 0; s < kSlots; ++s) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float x = __uint_as_float(sr[s][c]);
              const float e = (m_use == -INFINITY) ? 0.f : fast_exp2(x - m_use);
              sr[s][c] = __float_as_uint(e);
              rs += e;
            }
          }
          l = l * alpha + rs;
          m = m_use;
          // The previous PV must be done before P is overwritten or O rescaled.
          if (it > g0 && !warp_wait(bar_o_done, (it - 1) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (warp_need && it > g0) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(t_row + C::kOCol + c * 32, o);
              tmem_wait_ld();
              reg_fence32(o);
#pragma unroll
              for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
              tmem_st32(t_row + C::kOCol + c * 32, o);
            }
            tmem_wait_st();
          }
          // P (bf16) -> shared memory, K-major 128-byte swizzle, keys 0..127 in two panels.
#pragma unroll
          for (int s = 0; s < kSlots; ++s) {
            if (s >= ns) continue;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {   // 8 keys per 16-byte chunk
              const int key0 = s * 32 + ch * 8;
              const int pnl = key0 >> 6;
              const int cc = (key0 & 63) >> 3;
              uint32_t w0 = pack_bf16x2(__uint_as_float(sr[s][ch * 8 + 0]), __uint_as_float(sr[s][ch * 8 + 1]));
              uint32_t w1 = pack_bf16x2(__uint_as_float(sr[s][ch * 8 + 2]), __uint_as_float(sr[s][ch * 8 + 3]));
              uint32_t w2 = pack_bf16x2(__uint_as_float(sr[s][ch * 8 + 4]), __uint_as_float(sr[s][ch * 8 + 5]));
              uint32_t w3 = pack_bf16x2(__uint_as_float(sr[s][ch * 8 + 6]), __uint_as_float(sr[s][ch * 8 + 7]));
              const uint32_t addr = sP + pnl * kPanelBytes + r * kPanelRowBytes + ((cc ^ (r & 7)) << 4);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w0), "r"(w1),
                           "r"(w2), "r"(w3)
                           : "memory");
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(bar_p_full);
        }
        ++it;
        if (last) break;
      }
      if (!ok) break;

      if (C::kAttn) {
        // ---------------- epilogue: O / l -> bf16 -> smem (reuses the Q tile) -> TMA store
        if (!warp_wait(bar_o_done, (it - 1) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float inv_l = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_row + C::kOCol + c * 32, o);
          tmem_wait_ld();
          reg_fence32(o);
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const int col0 = c * 32 + ch * 8;
            const int pnl = col0 >> 6;
            const int cc = (col0 & 63) >> 3;
            uint32_t w[4];
#pragma unroll
            for (int x = 0; x < 4; ++x)
              w[x] = pack_bf16x2(__uint_as_float(o[ch * 8 + 2 * x]) * inv_l,
                                 __uint_as_float(o[ch * 8 + 2 * x + 1]) * inv_l);
            const uint32_t addr = sQ + pnl * kPanelBytes + r * kPanelRowBytes + ((cc ^ (r & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]), "r"(w[1]),
                         "r"(w[2]), "r"(w[3])
                         : "memory");
          }
        }
        if (p.lse != nullptr && i < p.n)
          p.lse[(long long)bh * p.n + i] =
              l > 0.f ? (m + __log2f(l)) * 0.6931471805599453f : -INFINITY;
        tc_fence_before();
        fence_proxy_async_smem();
        mbar_arrive(bar_o_staged);
        if (warp == 2 && lane == 0) {
          if (!mbar_wait(bar_o_staged, tl & 1, abort_flag, p.status)) {
            ok = false;
          } else {
            for (int pn = 0; pn < C::kPanels; ++pn)
              tma_store_3d(&tmO, sQ + pn * kPanelBytes, pn * 64, Qt * kBM, bh);
            bulk_commit_group();
            bulk_wait_group_read0();
            mbar_arrive(bar_q_empty);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) *abort_flag = 1;
      }
    }
    if (C::kAttn && warp == 2 && lane == 0) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---------------------------------------------------------------- host launchers

template <int D, int MODE>
static cudaError_t launch_impl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& to, const AttnParams& p, int grid,
                               cudaStream_t stream) {
  using C = Cfg<D, MODE>;
  static bool configured = false;  // per instantiation; attribute is per function
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<D, MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  attn_kernel<D, MODE><<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, to, p);
  return cudaGetLastError();
}

template <int MODE>
static cudaError_t launch_mode(int d, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const CUtensorMap& to, const AttnParams& p,
                               int grid, cudaStream_t stream) {
  switch (d) {
    case 64: return launch_impl<64, MODE>(tq, tk, tv, to, p, grid, stream);
    case 96: return launch_impl<96, MODE>(tq, tk, tv, to, p, grid, stream);
    case 128: return launch_impl<128, MODE>(tq, tk, tv, to, p, grid, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attention(int mode, int d, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, const CUtensorMap& to, const AttnParams& p,
                             int grid, cudaStream_t stream) {
  switch (mode) {
    case kModeDense: return launch_mode<kModeDense>(d, tq, tk, tv, to, p, grid, stream);
    case kModeSparse: return launch_mode<kModeSparse>(d, tq, tk, tv, to, p, grid, stream);
    case kModeMass: return launch_mode<kModeMass>(d, tq, tk, tv, to, p, grid, stream);
  }
  return cudaErrorInvalidValue;
}

int attention_smem_bytes(int mode, int d) {
  auto pick = [&](auto tag) { return decltype(tag)::kSmemBytes; };
  if (mode == kModeMass) {
    if (d == 64) return pick(Cfg<64, kModeMass>{});
    if (d == 96) return pick(Cfg<96, kModeMass>{});
    return pick(Cfg<128, kModeMass>{});
  }
  if (d == 64) return pick(Cfg<64, kModeDense>{});
  if (d == 96) return pick(Cfg<96, kModeDense>{});
  return pick(Cfg<128, kModeDense>{});
}

}  // namespace wise
