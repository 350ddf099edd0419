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
// Shared memory (128-byte swizzle, 1024-byte aligned panels of 64 columns):
//   Q tile [128 x d], K and V stage rings [128 keys x d], P [128 x 128] bf16.
// Tensor memory: S double buffer (2 x 128 fp32 columns) + one O accumulator
// per softmax half (2 x 128 columns).  Each half writes its P (bf16, two per
// column) over the first 32 columns of its own 64-column part of the S buffer
// it just read, and the PV MMA reads P from there (A operand in TMEM).

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100.cuh"
#include "wise_internal.h"

namespace wise {

constexpr int kBM = 128;        // query rows per tile
constexpr int kSlots = 4;       // key blocks per iteration
constexpr int kThreads = 352;   // 11 warps
constexpr int kPanelRowBytes = 128;                // 64 bf16 per swizzled row
constexpr int kPanelBytes = kBM * kPanelRowBytes;  // one 128-row panel = 16 KB
constexpr int kMaxWords = 16;   // schedule bitmask words per query block (nq <= 512)
constexpr int kInfoRing = 8;    // iterations of slot info in flight
constexpr int kSoftmaxThreads = 256;  // two halves of 4 warps

template <int D, int MODE>
struct Cfg {
  static constexpr int kPanels = (D + 63) / 64;
  static constexpr bool kAttn = MODE != kModeMass;
  static constexpr int kTileBytes = kPanels * kPanelBytes;  // Q tile, one K or V stage
  // K ring (freed when QK finishes) and V ring (freed when PV finishes).
  static constexpr int kKStages = kAttn ? (D <= 64 ? 4 : 3) : 4;
  static constexpr int kVStages = kAttn ? (D <= 64 ? 4 : 2) : 0;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffX = kOffV + kVStages * kTileBytes;   // epilogue (m, l) exchange
  static constexpr int kOffInfo = kOffX + (kAttn ? 2 * kBM * 8 : 0);
  static constexpr int kInfoBytes = 64;
  static constexpr int kOffMask = kOffInfo + kInfoRing * kInfoBytes;
  static constexpr int kOffBar = kOffMask + 4 * kMaxWords * 4;
  static constexpr int kVRing = kVStages > 0 ? kVStages : 1;  // barrier slots (mass mode: unused)
  // q_full, q_empty, k_full[K], k_empty[K], v_full[V], v_empty[V], info_full[I], info_empty[I],
  // s_full[2], s_free[2], p_full[2 halves][2 S buffers], o_done[2], merge, o_staged, final
  static constexpr int kNumBars = 2 + 2 * kKStages + 2 * kVRing + 2 * kInfoRing + 14;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = kAttn ? 512 : 256;
  static constexpr uint32_t kOCol = 256;   // O of half h at kOCol + 128 * h
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kInfoRing >= kKStages + 1, "info slot reuse needs QK of its iteration done");
};

struct StageInfo {
  int nslots;
  int last;
  int bh;
  int pad;
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
  __device__ bool empty() const { return next >= end; }
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
  __device__ bool empty() const {
    MaskList t = *this;
    while (t.cur == 0) {
      if (++t.w >= t.words) return true;
      t.cur = t.mask[t.w] | t.mask[kMaxWords + t.w] | t.mask[2 * kMaxWords + t.w] |
              t.mask[3 * kMaxWords + t.w];
    }
    return false;
  }
  __device__ bool pop(int& kb, int& own) {
    while (cur == 0) {
      if (++w >= words) return false;
      cur = mask[w] | mask[kMaxWords + w] | mask[2 * kMaxWords + w] | mask[3 * kMaxWords + w];
    }
    const int bit = __ffs(cur) - 1;
    cur &= cur - 1;
    kb = w * 32 + bit;
    own = 0;
#pragma unroll
    for (int r = 0; r < 4; ++r)
      if ((mask[r * kMaxWords + w] >> bit) & 1u) own |= 1 << r;
    return true;
  }
};

// Build the 4 per-row bitmasks of a sparse tile (whole producer warp).  Entries
// outside [0, q] or outside col_idx[0, col_count) are dropped and flagged.
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

template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
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
//
// Warp roles (352 threads): warp 0 = Q/K TMA producer and slot-list writer;
// warp 1 = TMEM allocator + single-thread MMA issuer; warp 2 = V TMA producer;
// warps 3..10 = softmax in two halves.  Half h (warps 3+4h .. 6+4h) owns key
// slots 2h and 2h+1 of every iteration (S columns 64h..64h+63)
// and keeps its own online-softmax state (m, l) and its own O accumulator in
// TMEM; the two partial results of a row are merged once, in the epilogue:
//   O = (2^(m_a-m) O_a + 2^(m_b-m) O_b) / (2^(m_a-m) l_a + 2^(m_b-m) l_b).
// Warp w reads TMEM lane quarter w % 4 (rows 32*(w%4) .. +31), i.e. one query
// block of the tile per warp.

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                const AttnParams p) {
  using C = Cfg<D, MODE>;
  constexpr int NK = C::kKStages;
  constexpr int NV = C::kVRing;  // mass mode has no V ring; its barrier slots stay unused
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t sQ = smem_u32(smem + C::kOffQ);
  const uint32_t sK = smem_u32(smem + C::kOffK);
  const uint32_t sV = smem_u32(smem + C::kOffV);
  StageInfo* info = (StageInfo*)(smem + C::kOffInfo);
  uint32_t* tile_mask = (uint32_t*)(smem + C::kOffMask);
  const uint32_t bar0 = smem_u32(smem + C::kOffBar);
  const uint32_t bar_q_full = bar0;
  const uint32_t bar_q_empty = bar0 + 8;
  const uint32_t barK = bar0 + 16;
  auto bar_k_full = [&](int s) { return barK + 8 * s; };
  auto bar_k_empty = [&](int s) { return barK + 8 * NK + 8 * s; };
  const uint32_t barV = barK + 16 * NK;
  auto bar_v_full = [&](int s) { return barV + 8 * s; };
  auto bar_v_empty = [&](int s) { return barV + 8 * NV + 8 * s; };
  const uint32_t barI = barV + 16 * NV;
  auto bar_i_full = [&](int s) { return barI + 8 * s; };
  auto bar_i_empty = [&](int s) { return barI + 8 * kInfoRing + 8 * s; };
  const uint32_t barS = barI + 16 * kInfoRing;
  auto bar_s_full = [&](int b) { return barS + 8 * b; };
  auto bar_s_free = [&](int b) { return barS + 16 + 8 * b; };
  // one p_full per (half, S buffer): the softmax may run an iteration ahead of the
  // MMA issuer, so a single barrier per half could complete two phases unobserved
  auto bar_p_full = [&](int h, int b) { return barS + 32 + 16 * h + 8 * b; };
  // one o_done per S buffer: arrives when both halves' PV of an iteration using that
  // buffer has completed (phase index = iteration >> 1)
  auto bar_o_done = [&](int b) { return barS + 64 + 8 * b; };
  const uint32_t bar_merge = barS + 80;
  const uint32_t bar_o_staged = barS + 88;
  const uint32_t bar_final = barS + 96;
  volatile int* abort_flag = (volatile int*)(smem + C::kOffMisc);
  uint32_t* tmem_slot = (uint32_t*)(smem + C::kOffMisc + 4);

  const int ntq = (p.nq + 3) / 4;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(bar_k_full(s), 1);
      mbar_init(bar_k_empty(s), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(bar_v_full(s), 1);
      mbar_init(bar_v_empty(s), 1);
    }
    for (int s = 0; s < kInfoRing; ++s) {
      mbar_init(bar_i_full(s), 1);
      // read by the 256 softmax threads and, in attention modes, the V producer
      mbar_init(bar_i_empty(s), kSoftmaxThreads + (C::kAttn ? 1 : 0));
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_s_full(b), 1);
      mbar_init(bar_s_free(b), kSoftmaxThreads);
      mbar_init(bar_p_full(0, b), kSoftmaxThreads / 2);
      mbar_init(bar_p_full(1, b), kSoftmaxThreads / 2);
      mbar_init(bar_o_done(b), 1);
    }
    mbar_init(bar_merge, kSoftmaxThreads);
    mbar_init(bar_o_staged, kSoftmaxThreads);
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
    // ======================================================= Q / K producer, slot lists
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
    }
    uint32_t it = 0;
    int tl = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tl) {
      int bh, Qt;
      decode_tile(tile, p.BH, ntq, bh, Qt);
      if (MODE == kModeSparse) build_tile_masks(tile_mask, p, bh, Qt, lane);
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
          int kbv[kSlots], ownv[kSlots];
          int n = 0;
          int kb, own;
          while (n < kSlots && (MODE == kModeSparse ? ml.pop(kb, own) : dl.pop(kb, own))) {
            kbv[n] = kb;
            ownv[n] = own;
            ++n;
          }
          if (n == 0) {
            if (!first) break;  // unreachable: `last` was set on the previous group
            kbv[0] = 0;         // empty tile: one fully masked slot keeps the pipeline uniform
            ownv[0] = 0;
            n = 1;
          }
          const bool last = (MODE == kModeSparse) ? ml.empty() : dl.empty();
          const int is = it % kInfoRing;
          if (it >= (uint32_t)kInfoRing &&
              !mbar_wait(bar_i_empty(is), ((it / kInfoRing) - 1) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          StageInfo& si = info[is];
          si.nslots = n;
          si.last = last ? 1 : 0;
          si.bh = bh;
          for (int s = 0; s < kSlots; ++s) {
            si.kb[s] = s < n ? kbv[s] : 0;
            si.own[s] = s < n ? ownv[s] : 0;
          }
          mbar_arrive(bar_i_full(is));
          const int ks = it % NK;
          if (it >= (uint32_t)NK &&
              !mbar_wait(bar_k_empty(ks), ((it / NK) - 1) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_k_full(ks), (uint32_t)n * 32 * kPanelRowBytes * C::kPanels);
          const uint32_t kbase = sK + ks * C::kTileBytes;
          for (int s = 0; s < n; ++s)
            for (int pn = 0; pn < C::kPanels; ++pn)
              tma_load_3d(kbase + pn * kPanelBytes + s * 32 * kPanelRowBytes, &tmK, bar_k_full(ks),
                          pn * 64, kbv[s] * 32, bh);
          ++it;
          first = false;
          if (last) break;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      it = __shfl_sync(0xffffffffu, it, 0);
    }
    if (lane == 0) {  // let the last K loads land before the CTA can exit
      const uint32_t from = it > (uint32_t)NK ? it - NK : 0u;
      for (uint32_t j = from; j < it; ++j) {
        volatile int dummy = 0;
        mbar_wait(bar_k_full(j % NK), (j / NK) & 1, &dummy, p.status);
      }
    }
  } else if (warp == 2) {
    // ======================================================= V producer (attention modes)
    if (C::kAttn && lane == 0) {
      tma_prefetch_desc(&tmV);
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        while (true) {
          const int is = it % kInfoRing;
          if (!mbar_wait(bar_i_full(is), (it / kInfoRing) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const int n = info[is].nslots;
          const int last = info[is].last;
          const int bh = info[is].bh;
          int kbv[kSlots];
#pragma unroll
          for (int s = 0; s < kSlots; ++s) kbv[s] = info[is].kb[s];
          mbar_arrive(bar_i_empty(is));
          const int vs = it % NV;
          if (it >= (uint32_t)NV &&
              !mbar_wait(bar_v_empty(vs), ((it / NV) - 1) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_v_full(vs), (uint32_t)n * 32 * kPanelRowBytes * C::kPanels);
          const uint32_t vbase = sV + vs * C::kTileBytes;
          for (int s = 0; s < n; ++s)
            for (int pn = 0; pn < C::kPanels; ++pn)
              tma_load_3d(vbase + pn * kPanelBytes + s * 32 * kPanelRowBytes, &tmV, bar_v_full(vs),
                          pn * 64, kbv[s] * 32, bh);
          ++it;
          if (last) break;
        }
      }
      const uint32_t from = it > (uint32_t)NV ? it - NV : 0u;
      for (uint32_t j = from; j < it; ++j) {
        volatile int dummy = 0;
        mbar_wait(bar_v_full(j % NV), (j / NV) & 1, &dummy, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================================================= MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);
      uint32_t it = 0;
      int tl = 0;
      bool ok = true;
      bool issued = false;
      // S_j = Q K_j^T into S buffer j&1; returns the iteration's slot count and last flag.
      auto issue_qk = [&](uint32_t j, int& ns, int& last) -> bool {
        const int ks = j % NK;
        if (!mbar_wait(bar_k_full(ks), (j / NK) & 1, abort_flag, p.status)) return false;
        if (j >= 2) {
          // S buffer j&1 still holds S_{j-2} (mass mode) or P_{j-2} (attention modes)
          if (!C::kAttn) {
            if (!mbar_wait(bar_s_free(j & 1), ((j >> 1) - 1) & 1, abort_flag, p.status))
              return false;
          } else if (!mbar_wait(bar_o_done(j & 1), ((j >> 1) - 1) & 1, abort_flag, p.status)) {
            return false;   // PV_{j-2} has read its P out of buffer j&1
          }
        }
        tc_fence_after();
        ns = info[j % kInfoRing].nslots;
        last = info[j % kInfoRing].last;
        const uint32_t idesc = idesc_bf16_f32(128, 32 * ns, 0, 0);
        const uint32_t d_tmem = tmem_base + (j & 1) * 128;
        const uint32_t kbase = sK + ks * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kPanelBytes + (kk & 3) * 32;
          mma_bf16_ss(d_tmem, smem_desc_sw128(sQ + off, 16, 1024),
                      smem_desc_sw128(kbase + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_s_full(j & 1));
        mma_commit(bar_k_empty(ks));
        issued = true;
        return true;
      };
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tl) {
        if (!mbar_wait(bar_q_full, tl & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        bool started[2] = {false, false};  // has half h's O been written in this tile
        int ns = 0, last = 1;
        if (!issue_qk(it, ns, last)) {
          ok = false;
          break;
        }
        while (true) {
          int ns_next = 0, last_next = 1;
          if (!last && !issue_qk(it + 1, ns_next, last_next)) {
            ok = false;
            break;
          }
          if (C::kAttn) {
            const int vs = it % NV;
            if (!mbar_wait(bar_v_full(vs), (it / NV) & 1, abort_flag, p.status)) {
              ok = false;
              break;
            }
            const uint32_t vbase = sV + vs * C::kTileBytes;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (!mbar_wait(bar_p_full(h, it & 1), (it >> 1) & 1, abort_flag, p.status)) {
                ok = false;
                break;
              }
              tc_fence_after();
              // half h: keys 64h .. 64h+63 of the iteration = 16-key steps 4h .. 4h+3;
              // its P sits in TMEM columns 64h .. 64h+31 of S buffer it&1 (8 per step)
              const int kend = min(2 * ns, 4 * h + 4);
              const uint32_t p_tmem = tmem_base + (it & 1) * 128 + 64 * h;
              for (int kk = 4 * h; kk < kend; ++kk) {
                const uint64_t b =
                    smem_desc_sw128(vbase + kk * 16 * kPanelRowBytes, kPanelBytes, 1024);
                mma_bf16_ts(tmem_base + C::kOCol + 128 * h, p_tmem + (kk - 4 * h) * 8, b, idesc_o,
                            (started[h] || kk > 4 * h) ? 1u : 0u);
              }
              if (kend > 4 * h) started[h] = true;
            }
            if (!ok) break;
            mma_commit(bar_o_done(it & 1));
            mma_commit(bar_v_empty(vs));
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
    // ======================================================= softmax / epilogue (warps 3..10)
    const int half = (warp - 3) >> 2;   // key slots 2*half, 2*half+1
    const int wg = warp & 3;            // TMEM lane quarter owned by this warp
    const int r = wg * 32 + lane;       // row within the tile
    const uint32_t t_row = tmem_base + ((uint32_t)(wg * 32) << 16);
    const uint32_t o_col = C::kOCol + 128 * half;
    const float sl2 = p.scale_log2;
    float* xchg = reinterpret_cast<float*>(smem + C::kOffX);
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
      bool started = false;   // mirrors the MMA issuer: this half's O written in this tile
      bool wrote_other = false;
      while (true) {
        const int is = it % kInfoRing;
        if (!warp_wait(bar_i_full(is), (it / kInfoRing) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        const int ns = info[is].nslots;
        const int last = info[is].last;
        int kbs[2], vld[2];
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int s = 2 * half + x;
          kbs[x] = info[is].kb[s];
          vld[x] = (s < ns) && ((info[is].own[s] >> wg) & 1);
        }
        mbar_arrive(bar_i_empty(is));
        if (!warp_wait(bar_s_full(it & 1), (it >> 1) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[2][32];
#pragma unroll
        for (int x = 0; x < 2; ++x)
          if (vld[x]) tmem_ld32(t_row + (it & 1) * 128 + (2 * half + x) * 32, sr[x]);
        tmem_wait_ld();
        reg_fence(sr[0]);
        reg_fence(sr[1]);
        if (!C::kAttn) {
          tc_fence_before();
          mbar_arrive(bar_s_free(it & 1));
          // ---------------- block mass: sum_j exp(s_ij*scale - lse_i) over the block, mean over rows
          float acc[2];
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            float a4[4] = {0.f, 0.f, 0.f, 0.f};
            if (vld[x]) {
              if (kbs[x] == qb) {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                  const float e = fast_exp2(fmaf(__uint_as_float(sr[x][c]), sl2, -lse_l2));
                  a4[c & 3] += (c > lane) ? 0.f : e;
                }
              } else {
#pragma unroll
                for (int c = 0; c < 32; ++c)
                  a4[c & 3] += fast_exp2(fmaf(__uint_as_float(sr[x][c]), sl2, -lse_l2));
              }
            }
            acc[x] = (a4[0] + a4[1]) + (a4[2] + a4[3]);
          }
          // the warp's 32 lanes are the 32 rows of query block qb: two interleaved butterflies
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], o);
            acc[1] += __shfl_xor_sync(0xffffffffu, acc[1], o);
          }
          if (lane < 2) {
            const float mine = lane == 0 ? acc[0] : acc[1];
            const int kbl = lane == 0 ? kbs[0] : kbs[1];
            const int v = lane == 0 ? vld[0] : vld[1];
            if (v) p.mass[((long long)bh * p.nq + qb) * p.nq + kbl] = mine * (1.0f / 32.0f);
          }
        } else {
          // ---------------- online softmax of this half (log2 domain, lazily rescaled)
          // Slot validity and the diagonal are warp-uniform branches.  Packed f32x2
          // FMA/ADD and 3-input max keep the instruction count per element low.
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if (vld[x] && kbs[x] == qb) {
#pragma unroll
              for (int c = 0; c < 32; ++c)
                if (c > lane) sr[x][c] = __float_as_uint(-INFINITY);
            }
          }
          float mxa[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if (vld[x]) {
#pragma unroll
              for (int c = 0; c < 32; c += 8) {
#pragma unroll
                for (int y = 0; y < 4; ++y)
                  mxa[y] = max3(mxa[y], __uint_as_float(sr[x][c + 2 * y]),
                                __uint_as_float(sr[x][c + 2 * y + 1]));
              }
            }
          }
          const float mx = max3(mxa[0], mxa[1], fmaxf(mxa[2], mxa[3])) * sl2;
          const float m_new = fmaxf(m, mx);
          const bool need = m_new > m + 8.0f;   // true on the first finite score
          const bool warp_need = __any_sync(0xffffffffu, need);
          const float m_use = warp_need ? m_new : m;
          const float alpha = (warp_need && m != -INFINITY) ? fast_exp2(m - m_use) : 1.0f;
          const float neg_m = (m_use == -INFINITY) ? 0.f : -m_use;  // all scores are -inf then
          const uint64_t sc2 = f2(sl2, sl2), nm2 = f2(neg_m, neg_m);
          float ps[2] = {0.f, 0.f};   // per-slot sums of this row's probabilities
          // P of slot x, keys 2c' and 2c'+1 as one bf16 pair, goes to sr[x][c'] (already consumed)
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if (vld[x]) {
              uint64_t rs2[2] = {0ull, 0ull};
#pragma unroll
              for (int c = 0; c < 32; c += 2) {
                float t0, t1;
                f2_split(fma2(f2(__uint_as_float(sr[x][c]), __uint_as_float(sr[x][c + 1])), sc2, nm2),
                         t0, t1);
                const float e0 = fast_exp2(t0), e1 = fast_exp2(t1);
                rs2[(c >> 1) & 1] = add2(rs2[(c >> 1) & 1], f2(e0, e1));
                sr[x][c >> 1] = pack_bf16x2(e0, e1);
              }
              float lo, hi;
              f2_split(add2(rs2[0], rs2[1]), lo, hi);
              ps[x] = lo + hi;
            } else {
#pragma unroll
              for (int c = 0; c < 16; ++c) sr[x][c] = 0u;   // not this warp's block: P = 0
            }
          }
          const float rs = ps[0] + ps[1];
          if (MODE == kModeDense && p.blse != nullptr) {
            // block log-sum-exp of this row over each owned key block, log2 domain:
            // blse = m + log2(sum_j 2^(s_ij*scale*log2e - m)); the mass pass turns it into
            // block mass with the final lse.  Layout [bh][key block][row]: 32 lanes store
            // 32 consecutive floats.
#pragma unroll
            for (int x = 0; x < 2; ++x) {
              if (vld[x])
                p.blse[((long long)bh * p.nq + kbs[x]) * p.n + i] =
                    ps[x] > 0.f ? m_use + __log2f(ps[x]) : -INFINITY;
            }
          }
          l = l * alpha + rs;
          m = m_use;
          if (warp_need && started) {
            // O of this half is rescaled in place: its previous PV must have finished.
            if (!warp_wait(bar_o_done((it - 1) & 1), ((it - 1) >> 1) & 1, abort_flag, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 16; ++c) {
              uint32_t o[16];
              tmem_ld16(t_row + o_col + c * 16, o);
              tmem_wait_ld();
              reg_fence(o);
#pragma unroll
              for (int y = 0; y < 16; ++y) o[y] = __float_as_uint(__uint_as_float(o[y]) * alpha);
              tmem_st16(t_row + o_col + c * 16, o);
            }
          }
          // P -> TMEM over the first 32 columns of this half's part of S buffer it&1
          tmem_st32_halves(t_row + (it & 1) * 128 + 64 * half, sr[0], sr[1]);
          tmem_wait_st();
          if (2 * ns > 4 * half) started = true;
          if (2 * ns > 4 * (1 - half)) wrote_other = true;
          tc_fence_before();
          mbar_arrive(bar_p_full(half, it & 1));
        }
        ++it;
        if (last) break;
      }
      if (!ok) break;

      if (C::kAttn) {
        // ---------------- epilogue: merge the halves, O -> bf16 -> smem (Q tile) -> TMA store
        if (!warp_wait(bar_o_done((it - 1) & 1), ((it - 1) >> 1) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // exchange (m, l) with the other half's thread of the same row (P buffer is idle now)
        xchg[(half * 128 + r) * 2 + 0] = m;
        xchg[(half * 128 + r) * 2 + 1] = l;
        mbar_arrive(bar_merge);
        if (!warp_wait(bar_merge, tl & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        const float m_o = xchg[((1 - half) * 128 + r) * 2 + 0];
        const float l_o = xchg[((1 - half) * 128 + r) * 2 + 1];
        const float ma = half == 0 ? m : m_o, la = half == 0 ? l : l_o;
        const float mb = half == 0 ? m_o : m, lb = half == 0 ? l_o : l;
        const bool a_written = half == 0 ? started : wrote_other;
        const bool b_written = half == 0 ? wrote_other : started;
        const float mt = fmaxf(ma, mb);
        const float sa = (la > 0.f) ? fast_exp2(ma - mt) : 0.f;
        const float sb = (lb > 0.f) ? fast_exp2(mb - mt) : 0.f;
        const float L = la * sa + lb * sb;
        const float inv = L > 0.f ? 1.0f / L : 0.f;
        const float ca = sa * inv, cb = sb * inv;
        // this half writes output columns [half*D/2, (half+1)*D/2)
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          const int col0 = half * (D / 2) + c * 16;
          uint32_t oa[16], ob[16];
#pragma unroll
          for (int y = 0; y < 16; ++y) oa[y] = ob[y] = 0u;
          if (a_written) tmem_ld16(t_row + C::kOCol + col0, oa);
          if (b_written) tmem_ld16(t_row + C::kOCol + 128 + col0, ob);
          tmem_wait_ld();
          reg_fence(oa);
          reg_fence(ob);
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            const int cabs = col0 + ch * 8;
            const int pnl = cabs >> 6;
            const int cc = (cabs & 63) >> 3;
            uint32_t w[4];
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              const int e0 = ch * 8 + 2 * y;
              const float v0 = __uint_as_float(oa[e0]) * ca + __uint_as_float(ob[e0]) * cb;
              const float v1 = __uint_as_float(oa[e0 + 1]) * ca + __uint_as_float(ob[e0 + 1]) * cb;
              w[y] = pack_bf16x2(v0, v1);
            }
            const uint32_t addr = sQ + pnl * kPanelBytes + r * kPanelRowBytes + ((cc ^ (r & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]), "r"(w[1]),
                         "r"(w[2]), "r"(w[3])
                         : "memory");
          }
        }
        if (half == 0 && p.lse != nullptr && i < p.n)
          p.lse[(long long)bh * p.n + i] =
              L > 0.f ? (mt + __log2f(L)) * 0.6931471805599453f : -INFINITY;
        tc_fence_before();
        fence_proxy_async_smem();
        mbar_arrive(bar_o_staged);
        if (warp == 3 && lane == 0) {
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
    if (C::kAttn && warp == 3 && lane == 0) bulk_wait_group0();
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
