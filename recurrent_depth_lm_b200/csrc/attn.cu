// attn.cu -- tcgen05/TMEM attention kernels of the WISE hot path (sm_100a).
//
// One persistent, warp-specialised kernel template covers four modes:
//   kDense    : exploration-step causal attention (all admissible key blocks), which
//               can also record per-(row, key block) log-sum-exps for the block mass,
//   kSparse   : late-step attention over a CSR key-block schedule,
//   kMass     : the block-mass pass with Q K^T recomputed (two-pass path; also the
//               16-token block mass),
//   kSparse16 : kSparse whose entries carry 16 x 16 sub-block masks (block size 16).
//
// Semantics follow Wan & Chen, "Attention Routing Stabilizes Early:
// Working-Set Inference for Recurrent-Depth Language Models": section 3
// (A = softmax(QK^T/sqrt(d_h) + M), O = AV), section 5.1 (block mass
// r_qb = mean over query rows of block q of the row's mass in key block b),
// section 5.2 (reuse mask: keys outside the working set are excluded) and
// section 7.4 (absent blocks are skipped; scoring, causal mask, online
// softmax and value aggregation are fused).
//
// Two query tiles in flight ("ping-pong").  A CTA keeps two tile slots
// X = 0, 1.  Each slot holds a 128-row query tile (4 query blocks of 32 rows),
// its own S region and O accumulator in tensor memory, and its own softmax
// warpgroup, which owns whole 128-key rows.  Per slot the work is a chain
//   QK_X(j) -> softmax_X(j) -> PV_X(j) -> QK_X(j+1)
// (S_X is reused, and P_X lives in S_X), so one slot alone would leave the
// tensor core idle during its softmax.  The single MMA thread therefore
// alternates between the slots -- PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1), ... --
// and the tensor core runs one slot's PV and QK while the other slot's softmax
// runs.  A slot that finishes its tile takes the CTA's next tile while the other
// slot keeps the tensor core busy; its output is written from registers, so the
// next query tile can be loaded as soon as the last QK of the previous one is done.
//
// Each iteration gathers up to 4 key blocks (128 keys) with one 32-row TMA box
// per block and panel, so a tile's key list may be any ascending set of blocks.
// A slot's "owner mask" says which of the tile's 4 query blocks may see a key
// block; rows of other query blocks get probability 0 for it.
//
// Shared memory (128-byte swizzle, 1024-byte aligned panels of 64 columns):
//   Q tiles [2][128 x d], K stage ring and V stage ring [128 keys x d] (both
//   filled in the CTA's global order of work entries), entry rings, masks.
// Tensor memory: S_X = columns [128 X, 128 X + 128); O_X = [256 + 128 X, +d).
// P_X (bf16, two per column) is written over the first 64 columns of S_X.

#include <cuda.h>
#include <cuda_bf16.h>

#include <atomic>
#include <cstdint>

#include "sm100.cuh"
#include "wise_internal.h"

namespace wise {

constexpr int kBM = 128;        // query rows per tile
constexpr int kSlots = 4;       // key blocks per iteration
constexpr int kThreads = 384;   // 3 warpgroups
constexpr int kPanelRowBytes = 128;                // 64 bf16 per swizzled row
constexpr int kPanelBytes = kBM * kPanelRowBytes;  // one 128-row panel = 16 KB
constexpr int kMaxWords = 16;   // schedule bitmask words per query block (nq <= 512)
constexpr int kRing = 4;        // work entries in flight per tile slot

enum : int { kWork = 0, kEnd = 1 };
enum : int { kFirst = 1, kLast = 2 };

// One work entry of a tile slot: one iteration of up to 4 key blocks, or the
// end marker of the slot.  Written by the Q/K producer, read by the V
// producer, the MMA issuer and the slot's softmax warpgroup.
struct Entry {
  int kind;
  int flags;   // kFirst / kLast of the slot's current tile
  int ns;      // key blocks used (1..4)
  int bh;
  int Qt;
  int stage;   // index among the CTA's work entries: K ring = stage % NK, V ring = stage % NV
  int kvh;     // K/V head of bh (bh / group), computed once per tile
  int pad0;
  int kb[kSlots];
  int own[kSlots];
};
static_assert(sizeof(Entry) == 64, "entry layout");

template <int D, int MODE>
struct Cfg {
  static constexpr int kPanels = (D + 63) / 64;
  static constexpr bool kAttn = MODE != kModeMass;
  static constexpr int kTileBytes = kPanels * kPanelBytes;  // Q tile, one K or V stage
  // block-size-16 sparse mode: its sub-mask planes need the shared memory of one K stage
  static constexpr int kKStages =
      kAttn ? (D <= 64 ? 4 : (MODE == kModeSparse16 ? 2 : 3)) : (D <= 64 ? 6 : 4);
  static constexpr int kVStages = kAttn ? (D <= 64 ? 4 : 2) : 0;
  static constexpr int kVRing = kVStages > 0 ? kVStages : 1;  // barrier slots (mass mode: unused)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffEnt = kOffV + kVStages * kTileBytes;
  static constexpr int kOffMask = kOffEnt + 2 * kRing * (int)sizeof(Entry);
  // per slot: 4 row masks of kMaxWords words; sparse16 adds 16 sub-mask planes
  static constexpr int kMaskWords = (MODE == kModeSparse16 ? 20 : 4) * kMaxWords;
  static constexpr int kOffBar = kOffMask + 2 * kMaskWords * 4;
  // q_full[2], q_empty[2], k_full[K], k_empty[K], v_full[V], v_empty[V], e_full[2][R],
  // e_empty[2][R], s_full[2], s_free[2], p_full[2], o_done[2], o_free[2], final
  static constexpr int kNumBars = 4 + 2 * kKStages + 2 * kVRing + 4 * kRing + 11;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = kAttn ? 512 : 256;
  static constexpr uint32_t kOCol = 256;   // O of slot X at kOCol + 128 * X
  static_assert(kSmemBytes <= 232448, "shared memory budget");
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
  // Block size 16: own = the 16 sub-mask bits (row r, bit j) at bit 4 r + j, read from
  // the planes by lanes 0..15 at once (whole warp, converged).
  __device__ bool pop_sub(int& kb, int& own, int lane) {
    while (cur == 0) {
      if (++w >= words) return false;
      cur = mask[w] | mask[kMaxWords + w] | mask[2 * kMaxWords + w] | mask[3 * kMaxWords + w];
    }
    const int bit = __ffs(cur) - 1;
    cur &= cur - 1;
    kb = w * 32 + bit;
    const bool set = lane < 16 && ((mask[(4 + lane) * kMaxWords + w] >> bit) & 1u);
    own = (int)(__ballot_sync(0xffffffffu, set) & 0xffffu);
    return true;
  }
};

// Build the 4 per-row bitmasks of a sparse tile (whole producer warp).  The tile's
// rows are consecutive in the CSR arrays: when their offsets are ascending within
// [0, col_count], one strided pass over col_idx[row_offsets[r0], row_offsets[r0 + nr])
// covers them.  Otherwise each row is taken on its own and a row with bad offsets
// is dropped.  Entries outside [0, q] are dropped.  Anything dropped is flagged.
//
// Block size 16 (kSub): entry e also carries p.sub[e], bit 2a + c = 16-row a of the
// query block keeps 16-column half c of the key block.  Bit j of row r goes to plane
// 4 r + j (mask + (4 + 4 r + j) * kMaxWords); an entry with no bit set is dropped.
template <bool kSub>
__device__ void build_tile_masks(uint32_t* mask, const AttnParams& p, int bh, int Qt, int lane) {
  const int words = (p.nq + 31) / 32;
  for (int x = lane; x < (kSub ? 20 : 4) * kMaxWords; x += 32) mask[x] = 0u;
  const int qb0 = Qt * 4;
  const int nr = min(4, p.nq - qb0);                 // rows of this tile
  const long long row0 = (long long)bh * p.nq + qb0;
  // offsets of rows r0 .. r0 + nr in lanes 0 .. nr (one load each)
  const long long off = lane <= nr ? (long long)p.row_offsets[row0 + lane] : 0;
  const long long o1 = __shfl_sync(0xffffffffu, off, min(1, nr));
  const long long o2 = __shfl_sync(0xffffffffu, off, min(2, nr));
  const long long o3 = __shfl_sync(0xffffffffu, off, min(3, nr));
  const long long nxt = __shfl_down_sync(0xffffffffu, off, 1);
  // lane r < nr checks row r: 0 <= beg <= end <= col_count
  const bool row_bad = lane < nr && (off < 0 || nxt < off || nxt > p.col_count);
  bool bad = false;
  __syncwarp();
  if (!__any_sync(0xffffffffu, row_bad)) {
    const long long beg = __shfl_sync(0xffffffffu, off, 0);
    const long long end = __shfl_sync(0xffffffffu, off, nr);
    // 8 entries per lane per round: all loads are issued before any is used
    for (long long e0 = beg + lane; e0 < end; e0 += 8 * 32) {
      int kbs[8];
      uint32_t subs[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const long long e = e0 + u * 32;
        kbs[u] = e < end ? p.col_idx[e] : 0;
        subs[u] = (kSub && e < end) ? (uint32_t)p.sub[e] & 15u : 15u;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const long long e = e0 + u * 32;
        if (e >= end) break;
        const int r = (e >= o1) + (e >= o2) + (e >= o3);   // row of entry e
        const int kb = kbs[u];
        if (kb >= 0 && kb <= qb0 + r && kb < words * 32) {
          if (subs[u] != 0u) atomicOr(&mask[r * kMaxWords + (kb >> 5)], 1u << (kb & 31));
          if (kSub) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if ((subs[u] >> j) & 1u)
                atomicOr(&mask[(4 + 4 * r + j) * kMaxWords + (kb >> 5)], 1u << (kb & 31));
          }
        } else {
          bad = true;
        }
      }
    }
  } else {
    bad = true;
    for (int r = 0; r < nr; ++r) {
      const long long beg = __shfl_sync(0xffffffffu, off, r);
      const long long end = __shfl_sync(0xffffffffu, nxt, r);
      if (__shfl_sync(0xffffffffu, row_bad ? 1 : 0, r)) continue;
      const int qb = qb0 + r;
      for (long long e = beg + lane; e < end; e += 32) {
        const int kb = p.col_idx[e];
        const uint32_t sb = kSub ? (uint32_t)p.sub[e] & 15u : 15u;
        if (kb >= 0 && kb <= qb && kb < words * 32 && sb != 0u) {
          atomicOr(&mask[r * kMaxWords + (kb >> 5)], 1u << (kb & 31));
          if (kSub) {
            for (int j = 0; j < 4; ++j)
              if ((sb >> j) & 1u)
                atomicOr(&mask[(4 + 4 * r + j) * kMaxWords + (kb >> 5)], 1u << (kb & 31));
          }
        }
      }
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.status, kStatusBadSchedule);
  __syncwarp();
}

// ---------------------------------------------------------------- helpers

template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// Block size 16: scores of the 16-column halves a row does not keep become -inf
// (keep bit c = columns 16 c .. 16 c + 15).
__device__ __forceinline__ void half_mask(uint32_t (&v)[32], uint32_t keep) {
#pragma unroll
  for (int c = 0; c < 32; ++c)
    if (!((keep >> (c >> 4)) & 1u)) v[c] = __float_as_uint(-INFINITY);
}

// kb[s] of a 4-entry register array for a runtime s, without local memory.
__device__ __forceinline__ int pick4(const int (&v)[4], int s) {
  return s == 0 ? v[0] : s == 1 ? v[1] : s == 2 ? v[2] : v[3];
}

// Warp-uniform bounded wait: every lane polls, the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          unsigned int* status) {
  bool ok = mbar_wait(bar, parity, abort, status);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) *abort = 1;
  return ok;
}

// The CTA's k-th tile: waves of gridDim.x tiles, every other wave in reverse CTA
// order, over tiles sorted heaviest first (largest Qt, most key blocks).
__device__ __forceinline__ int cta_tile(int k, int num_tiles) {
  const int G = gridDim.x;
  const int t = k * G + ((k & 1) ? (G - 1 - (int)blockIdx.x) : (int)blockIdx.x);
  return t < num_tiles ? t : -1;
}

__device__ __forceinline__ void decode_tile(int tile, int BH, int ntq, int& bh, int& Qt) {
  Qt = ntq - 1 - tile / BH;
  bh = tile % BH;
}

__device__ __forceinline__ void st_global_v4(void* ptr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(ptr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// ---------------------------------------------------------------- the kernel
//
// Warp roles (384 threads, 3 warpgroups):
//   warpgroup 0: warp 0 = Q/K TMA producer and entry writer (whole warp: sparse
//     masks), warp 1 = TMEM allocator + single-thread MMA issuer, warp 2 = V TMA
//     producer, warp 3 = idle;
//   warpgroup 1 (warps 4..7) = softmax of slot 0, warpgroup 2 (warps 8..11) =
//     softmax of slot 1.  Warp w reads TMEM lane quarter w % 4 (rows
//     32*(w%4) .. +31), i.e. one query block of its slot's tile; thread = row.
// Every party walks the two slot rings in the same order: alternate slots,
// skipping a slot once its end entry has been read.

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = Cfg<D, MODE>;
  constexpr int NK = C::kKStages;
  constexpr int NV = C::kVRing;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t sQ = smem_u32(smem + C::kOffQ);
  const uint32_t sK = smem_u32(smem + C::kOffK);
  const uint32_t sV = smem_u32(smem + C::kOffV);
  Entry* ents = (Entry*)(smem + C::kOffEnt);               // [2][kRing]
  uint32_t* masks = (uint32_t*)(smem + C::kOffMask);       // [2][kMaskWords]
  constexpr bool kSparseAny = MODE == kModeSparse || MODE == kModeSparse16;
  const uint32_t bar0 = smem_u32(smem + C::kOffBar);
  auto bar_q_full = [&](int x) { return bar0 + 8 * x; };
  auto bar_q_empty = [&](int x) { return bar0 + 16 + 8 * x; };
  const uint32_t barK = bar0 + 32;
  auto bar_k_full = [&](int s) { return barK + 8 * s; };
  auto bar_k_empty = [&](int s) { return barK + 8 * NK + 8 * s; };
  const uint32_t barV = barK + 16 * NK;
  auto bar_v_full = [&](int s) { return barV + 8 * s; };
  auto bar_v_empty = [&](int s) { return barV + 8 * NV + 8 * s; };
  const uint32_t barE = barV + 16 * NV;
  auto bar_e_full = [&](int x, int k) { return barE + 8 * (x * kRing + k); };
  auto bar_e_empty = [&](int x, int k) { return barE + 16 * kRing + 8 * (x * kRing + k); };
  const uint32_t barS = barE + 32 * kRing;
  auto bar_s_full = [&](int x) { return barS + 8 * x; };
  auto bar_s_free = [&](int x) { return barS + 16 + 8 * x; };   // mass mode: S read
  auto bar_p_full = [&](int x) { return barS + 32 + 8 * x; };   // P_X written
  auto bar_o_done = [&](int x) { return barS + 48 + 8 * x; };   // PV_X complete
  auto bar_o_free = [&](int x) { return barS + 64 + 8 * x; };   // O_X read by the epilogue
  const uint32_t bar_final = barS + 80;
  volatile int* abort_flag = (volatile int*)(smem + C::kOffMisc);
  uint32_t* tmem_slot = (uint32_t*)(smem + C::kOffMisc + 4);
  // abort flag of the drain waits at exit, which must not give up early
  volatile int* drain_flag = (volatile int*)(smem + C::kOffMisc + 8);

  const int ntq = (p.nq + 3) / 4;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *drain_flag = 0;
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar_q_full(x), 1);
      mbar_init(bar_q_empty(x), 1);
      for (int k = 0; k < kRing; ++k) {
        mbar_init(bar_e_full(x, k), 1);
        // read by the slot's 128 softmax threads, the MMA issuer and (attention) the V producer
        mbar_init(bar_e_empty(x, k), 128 + 1 + (C::kAttn ? 1 : 0));
      }
      mbar_init(bar_s_full(x), 1);
      mbar_init(bar_s_free(x), 128);
      mbar_init(bar_p_full(x), 128);
      mbar_init(bar_o_done(x), 1);
      mbar_init(bar_o_free(x), 128);
    }
    for (int s = 0; s < NK; ++s) {
      mbar_init(bar_k_full(s), 1);
      mbar_init(bar_k_empty(s), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(bar_v_full(s), 1);
      mbar_init(bar_v_empty(s), 1);
    }
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

  if (warp < 4) {
  if (warp == 0) {
    // ======================================================= Q / K producer, entry writer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
    }
    struct Slot {
      DenseList dl;
      MaskList ml;
      int bh, qt, rc, kvh;
      uint32_t tq;          // tiles started (q_empty phases)
      bool active, ended, first;
    };
    Slot sa{}, sb{};
    uint32_t g = 0;         // work entries written (K/V stage index)
    int next_k = 0;
    // One entry (work or end) for slot X; false on abort.
    auto step = [&](Slot& S, const int X) -> bool {
      const int k = S.rc % kRing;
      if (S.rc >= kRing &&
          !warp_wait(bar_e_empty(X, k), ((S.rc / kRing) - 1) & 1, abort_flag, p.status))
        return false;
      Entry& e = ents[X * kRing + k];
      if (!S.active) {
        const int tile = cta_tile(next_k++, p.num_tiles);
        if (tile < 0) {
          if (lane == 0) {
            e.kind = kEnd;
            mbar_arrive(bar_e_full(X, k));
          }
          ++S.rc;
          S.ended = true;
          return true;
        }
        decode_tile(tile, p.BH, ntq, S.bh, S.qt);
        S.kvh = S.bh / p.group;
        if (kSparseAny) {
          uint32_t* msk = masks + X * C::kMaskWords;
          build_tile_masks<MODE == kModeSparse16>(msk, p, S.bh, S.qt, lane);
          S.ml.init(msk, (p.nq + 31) / 32);
        } else {
          S.dl.init(S.qt, p.nq);
        }
        // the slot's previous tile must have finished its QK MMAs before Q_X is overwritten
        if (S.tq >= 1 && !warp_wait(bar_q_empty(X), (S.tq - 1) & 1, abort_flag, p.status))
          return false;
        if (lane == 0) {
          mbar_arrive_expect_tx(bar_q_full(X), C::kTileBytes);
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_3d(sQ + X * C::kTileBytes + pn * kPanelBytes, &tmQ, bar_q_full(X), pn * 64,
                        S.qt * kBM, S.bh);
        }
        ++S.tq;
        S.active = true;
        S.first = true;
      }
      int kbv[kSlots], ownv[kSlots];
      int n = 0;
      {
        int kb, own;
        while (n < kSlots && (MODE == kModeSparse16 ? S.ml.pop_sub(kb, own, lane)
                              : MODE == kModeSparse ? S.ml.pop(kb, own)
                                                    : S.dl.pop(kb, own))) {
          kbv[n] = kb;
          ownv[n] = own;
          ++n;
        }
      }
      if (n == 0) {  // empty tile: one fully masked key block keeps the pipeline uniform
        kbv[0] = 0;
        ownv[0] = 0;
        n = 1;
      }
      const bool last = kSparseAny ? S.ml.empty() : S.dl.empty();
      const int ks = g % NK;
      if (g >= (uint32_t)NK &&
          !warp_wait(bar_k_empty(ks), ((g / NK) - 1) & 1, abort_flag, p.status))
        return false;
      if (lane == 0) {
        e.kind = kWork;
        e.flags = (S.first ? kFirst : 0) | (last ? kLast : 0);
        e.ns = n;
        e.bh = S.bh;
        e.kvh = S.kvh;
        e.Qt = S.qt;
        e.stage = (int)g;
        for (int s = 0; s < kSlots; ++s) {
          e.kb[s] = s < n ? kbv[s] : 0;
          e.own[s] = s < n ? ownv[s] : 0;
        }
        mbar_arrive(bar_e_full(X, k));
        mbar_arrive_expect_tx(bar_k_full(ks), (uint32_t)n * 32 * kPanelRowBytes * C::kPanels);
        const uint32_t kbase = sK + ks * C::kTileBytes;
#pragma unroll 1
        for (int s = 0; s < n; ++s) {
          const int kb = pick4(kbv, s);
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_3d(kbase + pn * kPanelBytes + s * 32 * kPanelRowBytes, &tmK, bar_k_full(ks),
                        pn * 64, kb * 32, S.kvh);
        }
      }
      ++S.rc;
      ++g;
      S.first = false;
      if (last) S.active = false;
      return true;
    };
    // Alternate slots, skipping a slot that has ended.  One call site: the slot's
    // state is selected into S and written back (keeps the code compact).
    bool ok = true;
    for (int X = 0; ok && !(sa.ended && sb.ended); X ^= 1) {
      if (X == 0 ? sa.ended : sb.ended) continue;
      Slot S = X == 0 ? sa : sb;
      ok = step(S, X);
      if (X == 0) sa = S; else sb = S;
    }
    if (lane == 0) {  // let the last K and Q loads land before the CTA can exit
      const uint32_t from = g > (uint32_t)NK ? g - NK : 0u;
      for (uint32_t j = from; j < g; ++j) {
        mbar_wait(bar_k_full(j % NK), (j / NK) & 1, drain_flag, p.status);
      }
      if (sa.tq >= 1) mbar_wait(bar_q_full(0), (sa.tq - 1) & 1, drain_flag, p.status);
      if (sb.tq >= 1) mbar_wait(bar_q_full(1), (sb.tq - 1) & 1, drain_flag, p.status);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ======================================================= V producer (attention modes)
    if (C::kAttn && lane == 0) {
      tma_prefetch_desc(&tmV);
      struct Slot {
        int rc;
        bool ended;
      };
      Slot sa{}, sb{};
      uint32_t issued = 0;
      auto step = [&](Slot& S, const int X) -> bool {
        const int k = S.rc % kRing;
        if (!mbar_wait(bar_e_full(X, k), (S.rc / kRing) & 1, abort_flag, p.status)) return false;
        const Entry& e = ents[X * kRing + k];
        const int kind = e.kind;
        const int n = e.ns;
        const int kvh = e.kvh;
        const uint32_t g = (uint32_t)e.stage;
        int kbv[kSlots];
#pragma unroll
        for (int s = 0; s < kSlots; ++s) kbv[s] = e.kb[s];
        mbar_arrive(bar_e_empty(X, k));
        ++S.rc;
        if (kind == kEnd) {
          S.ended = true;
          return true;
        }
        const int vs = g % NV;
        if (g >= (uint32_t)NV &&
            !mbar_wait(bar_v_empty(vs), ((g / NV) - 1) & 1, abort_flag, p.status))
          return false;
        mbar_arrive_expect_tx(bar_v_full(vs), (uint32_t)n * 32 * kPanelRowBytes * C::kPanels);
        const uint32_t vbase = sV + vs * C::kTileBytes;
#pragma unroll 1
        for (int s = 0; s < n; ++s) {
          const int kb = pick4(kbv, s);
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_load_3d(vbase + pn * kPanelBytes + s * 32 * kPanelRowBytes, &tmV, bar_v_full(vs),
                        pn * 64, kb * 32, kvh);
        }
        issued = g + 1;
        return true;
      };
      bool ok = true;
      for (int X = 0; ok && !(sa.ended && sb.ended); X ^= 1) {
        if (X == 0 ? sa.ended : sb.ended) continue;
        Slot S = X == 0 ? sa : sb;
        ok = step(S, X);
        if (X == 0) sa = S; else sb = S;
      }
      const uint32_t from = issued > (uint32_t)NV ? issued - NV : 0u;
      for (uint32_t j = from; j < issued; ++j) {
        mbar_wait(bar_v_full(j % NV), (j / NV) & 1, drain_flag, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ======================================================= MMA issuer
    // The whole warp runs the issuer (converged, so its descriptor arithmetic stays
    // warp-uniform); one elected lane issues each MMA, commit and arrival.
    {
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);
      struct Slot {
        int rc;
        bool ended;
        bool pend;          // a work entry whose PV is not issued yet
        bool pend_first;
        int pend_ns, pend_stage;
        uint32_t pvc;       // PVs issued (p_full / o_done phases)
        uint32_t qkc;       // QKs issued (s_free phases)
        uint32_t qtiles;    // tiles whose first QK was issued (q_full phases)
        uint32_t otiles;    // tiles whose first PV was issued (o_free phases)
      };
      Slot sa{}, sb{};
      bool issued = false;

      // O_X (+)= P_X V of the slot's pending entry; P_X is read from TMEM (S_X columns).
      auto issue_pv = [&](Slot& S, const int X) -> bool {
        if (!warp_wait(bar_p_full(X), S.pvc & 1, abort_flag, p.status)) return false;
        if (S.pend_first) {
          // the first PV of a tile overwrites O_X: the previous tile's epilogue must have read it
          if (S.otiles >= 1 &&
              !warp_wait(bar_o_free(X), (S.otiles - 1) & 1, abort_flag, p.status))
            return false;
          ++S.otiles;
        }
        const uint32_t g = (uint32_t)S.pend_stage;
        const int vs = g % NV;
        if (!warp_wait(bar_v_full(vs), (g / NV) & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t vbase = sV + vs * C::kTileBytes;
        const uint32_t p_tmem = tmem_base + X * 128;
        const uint32_t o_tmem = tmem_base + C::kOCol + X * 128;
        const int nk = 2 * S.pend_ns;
        // descriptor start addresses advance by 16 keys = 2048 bytes (>> 4 = 128) per step
        const uint64_t b0 = smem_desc_sw128(vbase, kPanelBytes, 1024);
        for (int kk = 0; kk < nk; ++kk)
          mma_bf16_ts_warp(o_tmem, p_tmem + kk * 8, b0 + (uint64_t)(kk * 128), idesc_o,
                           (S.pend_first && kk == 0) ? 0u : 1u);
        mma_commit_warp(bar_o_done(X));
        mma_commit_warp(bar_v_empty(vs));
        ++S.pvc;
        S.pend = false;
        issued = true;
        return true;
      };

      // Read slot X's next entry: PV of its previous entry, then QK of this one.
      auto step = [&](Slot& S, const int X) -> bool {
        const int k = S.rc % kRing;
        if (!warp_wait(bar_e_full(X, k), (S.rc / kRing) & 1, abort_flag, p.status)) return false;
        const Entry& e = ents[X * kRing + k];
        const int kind = e.kind;
        const int flags = e.flags;
        const int ns = e.ns;
        const int stage = e.stage;
        __syncwarp();
        mbar_arrive_warp(bar_e_empty(X, k));
        ++S.rc;
        if (C::kAttn && S.pend && !issue_pv(S, X)) return false;
        if (kind == kEnd) {
          S.ended = true;
          return true;
        }
        // ---- S_X = Q_X K^T
        const int ks = stage % NK;
        if (!warp_wait(bar_k_full(ks), (stage / NK) & 1, abort_flag, p.status)) return false;
        if (flags & kFirst) {
          if (!warp_wait(bar_q_full(X), S.qtiles & 1, abort_flag, p.status)) return false;
          ++S.qtiles;
        }
        // Attention modes: S_X holds P_X, which the PV just issued reads.  tcgen05 MMAs
        // issued by one thread execute in issue order, so this QK overwrites S_X only
        // after that PV has read it, with no wait for the PV here; and the s_full commit
        // below tracks the PV too, so the softmax may rescale O_X once S_X is ready.
        // Mass mode: the softmax warps read S_X itself, so wait until they are done.
        if (!C::kAttn && S.qkc >= 1 &&
            !warp_wait(bar_s_free(X), (S.qkc - 1) & 1, abort_flag, p.status))
          return false;
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(128, 32 * ns, 0, 0);
        const uint32_t d_tmem = tmem_base + X * 128;
        const uint32_t qbase = sQ + X * C::kTileBytes;
        const uint32_t kbase = sK + ks * C::kTileBytes;
        // K steps of 16 columns: +32 bytes within a 64-column panel, then the next panel;
        // the descriptors' start fields (address >> 4) advance by the same offsets >> 4
        const uint64_t a0 = smem_desc_sw128(qbase, 16, 1024);
        const uint64_t b0 = smem_desc_sw128(kbase, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * kPanelBytes + (kk & 3) * 32) >> 4);
          mma_bf16_ss_warp(d_tmem, a0 + off, b0 + off, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit_warp(bar_s_full(X));
        mma_commit_warp(bar_k_empty(ks));
        if (flags & kLast) mma_commit_warp(bar_q_empty(X));  // Q_X may be reloaded
        ++S.qkc;
        issued = true;
        if (C::kAttn) {
          S.pend = true;
          S.pend_ns = ns;
          S.pend_stage = stage;
          S.pend_first = (flags & kFirst) != 0;
        }
        return true;
      };

      bool ok = true;
      for (int X = 0; ok && !(sa.ended && sb.ended); X ^= 1) {
        if (X == 0 ? sa.ended : sb.ended) continue;
        Slot S = X == 0 ? sa : sb;
        ok = step(S, X);
        if (X == 0) sa = S; else sb = S;
      }
      if (issued) {
        mma_commit_warp(bar_final);
        mbar_wait(bar_final, 0, drain_flag, p.status);
      }
      __syncwarp();
    }
  }
  } else {
    // ======================================================= softmax / epilogue of slot X
    // Thread = row.  Each iteration reads its key blocks from S_X once, one 32-column
    // block at a time in a rolled loop (block max, then exponentials against the row's
    // reference): the hot loop stays small enough for the instruction cache.
    const int X = (warp - 4) >> 2;
    const int qw = warp & 3;            // TMEM lane quarter = query block within the tile
    const uint32_t t_lane = tmem_base + ((uint32_t)(qw * 32) << 16);
    const uint32_t s_col = X * 128;
    const uint32_t o_col = C::kOCol + X * 128;
    const float sl2 = p.scale_log2;
    int rc = 0;
    uint32_t cnt = 0;                   // work entries processed (s_full / o_done phases)
    bool run = true;
    while (run) {
      // ---------------- one tile of the slot: its entries, then the epilogue
      float m = -INFINITY, l = 0.f, l32 = 0.f, lse_l2 = 0.f;
      int bh = 0, qb = 0, i = 0;
      bool first = true;
      while (true) {
        const int k = rc % kRing;
        if (!warp_wait(bar_e_full(X, k), (rc / kRing) & 1, abort_flag, p.status)) {
          run = false;
          break;
        }
        // The entry stays valid until this warp's arrival on e_empty at the end of
        // the iteration: key-block indices are read from it as needed.
        const Entry& e = ents[X * kRing + k];
        const int kind = e.kind;
        const int flags = e.flags;
        if (kind == kEnd) {
          mbar_arrive(bar_e_empty(X, k));
          ++rc;
          run = false;
          break;
        }
        const int ns = e.ns;
        uint32_t vmask = 0u, dmask = 0u;   // key blocks this row sees; diagonal blocks
        uint32_t hmask = 0u;               // block size 16: kept halves, 2 bits per block
        if (first) {
          bh = e.bh;
          qb = e.Qt * 4 + qw;
          i = qb * 32 + lane;
          if (!C::kAttn && qb < p.nq)
            lse_l2 = p.lse_in[(long long)bh * p.n + i] * 1.4426950408889634f;
        }
#pragma unroll
        for (int s = 0; s < kSlots; ++s) {
          if (MODE == kModeSparse16) {
            // own: bit 4 r + 2 a + c = 16-row a of query block r keeps half c
            const int o4 = s < ns ? (e.own[s] >> (4 * qw)) & 15 : 0;
            if (o4 != 0) {
              vmask |= 1u << s;
              if (e.kb[s] == qb) dmask |= 1u << s;
              hmask |= (uint32_t)((o4 >> (2 * (lane >> 4))) & 3) << (2 * s);
            }
          } else if (s < ns && ((e.own[s] >> qw) & 1)) {
            vmask |= 1u << s;
            if (e.kb[s] == qb) dmask |= 1u << s;
          }
        }
        if (!warp_wait(bar_s_full(X), cnt & 1, abort_flag, p.status)) {
          run = false;
          break;
        }
        tc_fence_after();
        ++cnt;

        if (!C::kAttn) {
          // -------- block mass: sum_j 2^(s_ij*scale*log2e - lse_i*log2e), mean over rows
#pragma unroll 1
          for (int s = 0; s < kSlots; ++s) {
            if (!((vmask >> s) & 1u)) continue;
            uint32_t v[32];
            tmem_ld32(t_lane + s_col + s * 32, v);
            tmem_wait_ld();
            reg_fence(v);
            const bool diag = (dmask >> s) & 1u;
            if (p.fine16) {
              // 16-token blocks: lanes 0..15 / 16..31 are 16-rows 2 qb / 2 qb + 1; a4[0..1]
              // would mix the halves, so sum each 16-column half on its own
              float lo = 0.f, hi = 0.f;
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                const float ev = fast_exp2(fmaf(__uint_as_float(v[c]), sl2, -lse_l2));
                const float x = (diag && c > lane) ? 0.f : ev;
                if (c < 16) lo += x; else hi += x;
              }
#pragma unroll
              for (int o = 8; o > 0; o >>= 1) {
                lo += __shfl_xor_sync(0xffffffffu, lo, o);
                hi += __shfl_xor_sync(0xffffffffu, hi, o);
              }
              if ((lane & 15) == 0) {
                const long long nq16 = 2ll * p.nq;
                float* dst = p.mass + ((long long)bh * nq16 + 2 * qb + (lane >> 4)) * nq16 +
                             2 * e.kb[s];
                dst[0] = lo * (1.0f / 16.0f);
                dst[1] = hi * (1.0f / 16.0f);
              }
              continue;
            }
            float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float ev = fast_exp2(fmaf(__uint_as_float(v[c]), sl2, -lse_l2));
              a4[c & 3] += (diag && c > lane) ? 0.f : ev;
            }
            // the warp's 32 lanes are the 32 rows of query block qb
            float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) p.mass[((long long)bh * p.nq + qb) * p.nq + e.kb[s]] = acc * (1.0f / 32.0f);
          }
          tc_fence_before();
          mbar_arrive(bar_s_free(X));
          mbar_arrive(bar_e_empty(X, k));
          ++rc;
          first = false;
          if (flags & kLast) break;
          continue;
        }

        // -------- one pass over the entry's key blocks: P = 2^(s*scale*log2e - m_ref) as
        // bf16 pairs over S_X columns [0, 64).  Key block s goes to P columns
        // [16 s, 16 s + 16), which lie below S block s: reading S block s never sees P.
        // m_ref is the row's exponent reference, an integer: it moves only when a block's
        // max exceeds it by more than 2^8, and then the P blocks already written (and the
        // row sums) are rescaled in place by an exact power of two, so every P of the
        // entry shares one reference and no value is rounded twice.
        // rs sums the fp32 P (it gives the log-sum-exps); rcorr adds, per key block, the
        // bf16 rounding error of the block's largest P.  O is normalised by rs + rcorr: the
        // PV MMA multiplies the bf16-rounded P into V, and where a few keys carry the
        // row's weight the rounding of those P is what would otherwise bias O.
        float m_ref = m;
        float rs = 0.f, rcorr = 0.f;
        const uint64_t sc2 = f2(sl2, sl2);
        auto rescale_p = [&](int s, float f) {
          tmem_wait_st();   // the P stores of the earlier blocks have landed
#pragma unroll 1
          for (int t = 0; t < s; ++t) {
            if (!((vmask >> t) & 1u)) continue;   // P = 0 there
            uint32_t w[16];
            tmem_ld16(t_lane + s_col + t * 16, w);
            tmem_wait_ld();
            reg_fence(w);
#pragma unroll
            for (int y = 0; y < 16; ++y) {
              const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[y]);
              w[y] = pack_bf16x2(__low2float(h) * f, __high2float(h) * f);
            }
            tmem_st16(t_lane + s_col + t * 16, w);
          }
        };
        auto block_exp = [&](uint32_t (&v)[32], int s) {
          uint32_t w[16];
          if ((vmask >> s) & 1u) {
            reg_fence(v);
            if ((dmask >> s) & 1u) {
#pragma unroll
              for (int c = 0; c < 32; ++c)
                if (c > lane) v[c] = __float_as_uint(-INFINITY);
            }
            if (MODE == kModeSparse16 && ((hmask >> (2 * s)) & 3u) != 3u)
              half_mask(v, (hmask >> (2 * s)) & 3u);
            float mxa[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
#pragma unroll
              for (int y = 0; y < 4; ++y)
                mxa[y] = max3(mxa[y], __uint_as_float(v[c + 2 * y]), __uint_as_float(v[c + 2 * y + 1]));
            }
            const float bmax = max3(mxa[0], mxa[1], fmaxf(mxa[2], mxa[3]));
            const float bm = bmax * sl2;
            const bool trig = bm > m_ref + 8.0f;   // true on the row's first finite score
            if (__any_sync(0xffffffffu, trig)) {
              const float m_new = trig ? ceilf(bm) : m_ref;
              const float f = trig ? exp2_int(m_ref - m_new) : 1.0f;   // 0 from -inf
              rescale_p(s, f);
              rs *= f;
              rcorr *= f;
              m_ref = m_new;
            }
            const float neg_m = (m_ref == -INFINITY) ? 0.f : -m_ref;  // all scores -inf then
            const uint64_t nm2 = f2(neg_m, neg_m);
            // Dense mode keeps the row sum of each 16-column half apart (the 16-token block
            // log-sum-exps); the 16-token sparse mode sums the same way, so that on an
            // all-blocks schedule it reproduces dense attention bit for bit; the 32-token
            // sparse mode needs only the block's sum.
            constexpr bool kHalves = MODE == kModeDense || MODE == kModeSparse16;
            uint64_t rs2[2][2] = {{0ull, 0ull}, {0ull, 0ull}};   // [16-column half][pair parity]
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              float t0, t1;
              f2_split(fma2(f2(__uint_as_float(v[c]), __uint_as_float(v[c + 1])), sc2, nm2), t0, t1);
              const float e0 = fast_exp2(t0), e1 = fast_exp2(t1);
              uint64_t& acc = rs2[kHalves ? (c >> 4) : 0][(c >> 1) & 1];
              acc = add2(acc, f2(e0, e1));
              w[c >> 1] = pack_bf16x2(e0, e1);
            }
            float ps16[2] = {0.f, 0.f};   // sums over columns 0..15 and 16..31 (dense mode)
            float ps;
            {
              float a0, a1;
              f2_split(add2(rs2[0][0], rs2[0][1]), a0, a1);
              if (kHalves) {
                float b0, b1;
                f2_split(add2(rs2[1][0], rs2[1][1]), b0, b1);
                ps16[0] = a0 + a1;
                ps16[1] = b0 + b1;
                ps = ps16[0] + ps16[1];
              } else {
                ps = a0 + a1;
              }
            }
            rs += ps;
            {
              // the block's largest P, computed as its element was, and its bf16 rounding
              const float pm = fast_exp2(fmaf(bmax, sl2, neg_m));
              rcorr += __uint_as_float(pack_bf16x2(pm, 0.f) << 16) - pm;
            }
            if (MODE == kModeDense && p.blse != nullptr) {
              // block log-sum-exp of this row over key block kb, log2 domain:
              // blse = m + log2(sum_j 2^(s_ij*scale*log2e - m)); the mass pass turns it
              // into block mass with the final lse.  Layout [bh][key block][row]: 32
              // lanes store 32 consecutive floats.  fine16: one value per 16-key half,
              // key block 2 kb + half of the 16-token blocks.
              if (p.fine16) {
                float* dst = p.blse + ((long long)bh * 2 * p.nq + 2 * e.kb[s]) * p.n + i;
                dst[0] = ps16[0] > 0.f ? m_ref + __log2f(ps16[0]) : -INFINITY;
                dst[p.n] = ps16[1] > 0.f ? m_ref + __log2f(ps16[1]) : -INFINITY;
              } else {
                p.blse[((long long)bh * p.nq + e.kb[s]) * p.n + i] =
                    ps > 0.f ? m_ref + __log2f(ps) : -INFINITY;
              }
            }
          } else {
#pragma unroll
            for (int c = 0; c < 16; ++c) w[c] = 0u;   // not this row's block (or unused): P = 0
          }
          tmem_st16(t_lane + s_col + s * 16, w);
        };
#pragma unroll 1
        for (int s = 0; s < kSlots; ++s) {
          uint32_t v[32];
          if ((vmask >> s) & 1u) {
            tmem_ld32(t_lane + s_col + s * 32, v);
            tmem_wait_ld();
          }
          block_exp(v, s);
        }
        const bool need = m_ref != m;   // this row's reference moved during the entry
        const bool warp_need = __any_sync(0xffffffffu, need);
        const float alpha = (need && m != -INFINITY) ? exp2_int(m - m_ref) : 1.0f;
        const float m_use = m_ref;
        if (warp_need && !first) {
          // O_X is rescaled in place.  Its last PV has completed: QK_X of this entry
          // was issued only after it.
#pragma unroll 1
          for (int c = 0; c < D / 16; ++c) {
            uint32_t o[16];
            tmem_ld16(t_lane + o_col + c * 16, o);
            tmem_wait_ld();
            reg_fence(o);
#pragma unroll
            for (int y = 0; y < 16; ++y) o[y] = __float_as_uint(__uint_as_float(o[y]) * alpha);
            tmem_st16(t_lane + o_col + c * 16, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_p_full(X));
        mbar_arrive(bar_e_empty(X, k));
        ++rc;
        l = l * alpha + (rs + rcorr);
        l32 = l32 * alpha + rs;
        m = m_use;
        first = false;
        if (flags & kLast) break;
      }
      if (!run || !C::kAttn) continue;

      // ---------------- epilogue: O_X / l -> bf16 -> global rows (one row per thread)
      if (!warp_wait(bar_o_done(X), (cnt - 1) & 1, abort_flag, p.status)) break;
      tc_fence_after();
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      if (qb < p.nq) {
        uint8_t* orow = static_cast<uint8_t*>(p.o) + ((long long)bh * p.n + i) * (D * 2);
#pragma unroll 1
        for (int c = 0; c < D / 16; ++c) {
          uint32_t o[16];
          tmem_ld16(t_lane + o_col + c * 16, o);
          tmem_wait_ld();
          reg_fence(o);
          uint32_t w[8];
#pragma unroll
          for (int y = 0; y < 8; ++y)
            w[y] = pack_bf16x2(__uint_as_float(o[2 * y]) * inv, __uint_as_float(o[2 * y + 1]) * inv);
          st_global_v4(orow + c * 32, w[0], w[1], w[2], w[3]);
          st_global_v4(orow + c * 32 + 16, w[4], w[5], w[6], w[7]);
        }
        if (p.lse != nullptr)
          p.lse[(long long)bh * p.n + i] =
              l32 > 0.f ? (m + __log2f(l32)) * 0.6931471805599453f : -INFINITY;
      }
      tc_fence_before();
      mbar_arrive(bar_o_free(X));
    }
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
                               const AttnParams& p, int grid, cudaStream_t stream,
                               const char** why) {
  using C = Cfg<D, MODE>;
  // The shared-memory limit is a per-device attribute of the function: set it once per
  // device (a repeated set from racing threads is harmless).
  constexpr int kDevs = 64;
  static std::atomic<bool> configured[kDevs];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kDevs) return cudaErrorInvalidDevice;
  if (!configured[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(attn_kernel<D, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev].store(true, std::memory_order_release);
  }
  attn_kernel<D, MODE><<<grid, kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

template <int MODE>
static cudaError_t launch_mode(int d, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const AttnParams& p, int grid,
                               cudaStream_t stream, const char** why) {
  switch (d) {
    case 64: return launch_impl<64, MODE>(tq, tk, tv, p, grid, stream, why);
    case 96: return launch_impl<96, MODE>(tq, tk, tv, p, grid, stream, why);
    case 128: return launch_impl<128, MODE>(tq, tk, tv, p, grid, stream, why);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_attention(int mode, int d, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, const AttnParams& p, int grid,
                             cudaStream_t stream, const char** why) {
  switch (mode) {
    case kModeDense: return launch_mode<kModeDense>(d, tq, tk, tv, p, grid, stream, why);
    case kModeSparse: return launch_mode<kModeSparse>(d, tq, tk, tv, p, grid, stream, why);
    case kModeMass: return launch_mode<kModeMass>(d, tq, tk, tv, p, grid, stream, why);
    case kModeSparse16: return launch_mode<kModeSparse16>(d, tq, tk, tv, p, grid, stream, why);
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
  if (mode == kModeSparse16) {
    if (d == 64) return pick(Cfg<64, kModeSparse16>{});
    if (d == 96) return pick(Cfg<96, kModeSparse16>{});
    return pick(Cfg<128, kModeSparse16>{});
  }
  if (d == 64) return pick(Cfg<64, kModeDense>{});
  if (d == 96) return pick(Cfg<96, kModeDense>{});
  return pick(Cfg<128, kModeDense>{});
}

}  // namespace wise
