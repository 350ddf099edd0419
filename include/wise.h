/*
 * wise.h -- C ABI of the WISE attention hot path on NVIDIA B200 (sm_100a).
 *
 * WISE ("Working-set Inference with Support Exploitation") is described in
 * Wan & Chen, "Attention Routing Stabilizes Early: Working-Set Inference for
 * Recurrent-Depth Language Models" (arXiv 2609.27373), "the WISE paper"
 * below.  One recurrent step of one attention layer goes through:
 *
 *   exploration steps t <= t_d : wise_full_attn_mass   (dense causal attention,
 *                                  plus block mass on discovery-window steps)
 *                                wise_select_union     (cumulative-eta support,
 *                                  OR-ed into the working set; or
 *                                  wise_select_union_blocks for B = 64 / 128;
 *                                  the *_b16 calls for B = 16)
 *                                wise_window_step      (a window step's attention,
 *                                  block mass and selection in one call, B = 32)
 *   once, after step t_d       : wise_build_schedule   (CSR key-block schedule)
 *   late steps t > t_d         : wise_sparse_attn      (block-sparse attention)
 *   analysis, off the hot path : wise_select_size_matched / _mass_matched
 *                                  (selection-only controls), wise_support_mass
 *                                  (retained attention mass of a support)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Block size B = 32 tokens (WISE paper section 7.1, "WISE configuration").
 * - Q, K, V, O are bf16, contiguous [batch, heads, seqlen, head_dim]
 *   (row-major, head_dim fastest).  head_dim is 64, 96 or 128; seqlen is a
 *   positive multiple of 32 and at most 16384.  nq = seqlen / 32 blocks.
 *   "BH" = batch * heads.  Q, K, V, O base addresses must be 16-byte aligned.
 * - All data pointers are DEVICE pointers allocated by the caller; the library
 *   allocates no device memory and never takes ownership.  Host pointers are
 *   marked as such.
 * - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *   enqueue work and return; the one exception is wise_build_schedule with a
 *   non-NULL nnz_out, which synchronises `stream`.
 * - Return value: WISE_OK (0) on success, a negative WISE_ERR_* otherwise.
 *   On error nothing is enqueued and wise_last_error() (thread-local) holds a
 *   message.  Faults detected on the device (an invalid schedule entry, or a
 *   pipeline wait that ran out of time) do not stop the kernel: they set bits
 *   in a device status word read by wise_device_status().
 */
#ifndef WISE_H_
#define WISE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WISE_OK 0
#define WISE_ERR_ARG (-1)      /* NULL pointer where one is required, bad eta */
#define WISE_ERR_SHAPE (-2)    /* unsupported head_dim / seqlen / sizes        */
#define WISE_ERR_ALIGN (-3)    /* pointer not 16-byte aligned                  */
#define WISE_ERR_CAPACITY (-4) /* col_idx too small for the schedule           */
#define WISE_ERR_CUDA (-5)     /* CUDA runtime or driver error                 */
#define WISE_ERR_WORKSPACE (-6)/* workspace missing or too small               */

/* Device status bits (wise_device_status). */
#define WISE_STATUS_TIMEOUT 0x1u        /* a bounded pipeline wait expired        */
#define WISE_STATUS_BAD_SCHEDULE 0x2u   /* schedule entry out of range / unsorted */

#define WISE_BLOCK 32

typedef struct wise_shape {
  int32_t batch;
  int32_t heads;
  int32_t seqlen;
  int32_t head_dim;
  float scale; /* softmax temperature; <= 0 selects 1/sqrt(head_dim) (WISE paper section 3) */
  /* Heads of K and V (grouped-query attention, as in the Recurrent-Llama geometry of the
   * WISE paper, section 4: 32 query heads over 8 key/value heads).  0 means kv_heads =
   * heads.  heads must be a multiple of kv_heads; query head h reads K/V head
   * h / (heads / kv_heads), and K, V are then [batch, kv_heads, seqlen, head_dim]. */
  int32_t kv_heads;
} wise_shape_t;

/*
 * Dense causal attention of one exploration step, optionally with block mass.
 *
 * Defines (WISE paper section 3, recurrent attention equation):
 *   A = softmax(Q K^T * scale + M),  O = A V,  M_ij = -inf for j > i.
 * and, when `mass` is non-NULL, the block mass of section 5.1:
 *   mass[bh][q][b] = (1/32) sum_{i in block q} sum_{j in block b} A_ij,  b <= q.
 *
 * q, k, v   : bf16 [B, H, n, d] inputs.
 * o         : bf16 [B, H, n, d] output.
 * lse       : fp32 [B, H, n] output, natural-log row normaliser
 *             lse_i = log sum_{j<=i} exp(s_ij * scale); may be NULL unless
 *             mass is requested.
 * mass      : fp32 [B, H, nq, nq] output or NULL.  Only entries b <= q are
 *             written; entries b > q are left untouched.
 * workspace : device scratch for the one-pass mass, or NULL.  With at least
 *             wise_mass_workspace_bytes(shape) bytes the attention kernel also
 *             records every row's per-key-block log-sum-exp and a light kernel
 *             turns them into block masses; with NULL the mass is computed by a
 *             second pass that recomputes Q K^T.  Ignored when mass is NULL.
 * Errors    : WISE_ERR_ARG (q/k/v/o NULL, mass without lse), WISE_ERR_SHAPE,
 *             WISE_ERR_ALIGN, WISE_ERR_WORKSPACE (non-NULL but too small),
 *             WISE_ERR_CUDA.
 */
int wise_full_attn_mass(const void* q, const void* k, const void* v, void* o, float* lse,
                        float* mass, void* workspace, size_t workspace_bytes, wise_shape_t shape,
                        void* stream);

/*
 * One step of the discovery window in one call: dense causal attention with lse, the
 * block mass and the step's cumulative-eta support ORed into the working set.
 *
 * Defines (WISE paper appendix B "WISE configuration": the window steps
 * t_d - 3 .. t_d; section 3 recurrent attention equation; section 5.1 block mass;
 * section 3 "attention support" and section 6.1 selection): exactly
 *   wise_full_attn_mass(q, k, v, o, lse, mass, workspace, ...) followed by
 *   wise_select_union(mass, union_bits, step_bits, eta, ...),
 * with the same outputs bit for bit: the attention kernel records every row's
 * per-key-block log-sum-exp in `workspace`, a light kernel turns them into block
 * masses and the selection kernel cuts each row at eta.
 *
 * q, k, v, o, lse, mass : as for wise_full_attn_mass; lse and mass are required.
 * union_bits, step_bits, eta : as for wise_select_union.
 * workspace  : device scratch of at least wise_mass_workspace_bytes(shape) bytes,
 *              16-byte aligned (required).
 * Errors     : WISE_ERR_ARG (a required pointer NULL, eta <= 0 or NaN), WISE_ERR_SHAPE,
 *              WISE_ERR_ALIGN, WISE_ERR_WORKSPACE (too small), WISE_ERR_CUDA.
 */
int wise_window_step(const void* q, const void* k, const void* v, void* o, float* lse,
                     float* mass, uint32_t* union_bits, uint32_t* step_bits, float eta,
                     void* workspace, size_t workspace_bytes, wise_shape_t shape, void* stream);

/* Workspace bytes of the one-pass block mass: B * H * nq * n * 4. */
size_t wise_mass_workspace_bytes(wise_shape_t shape);

/*
 * Per-step cumulative-eta block support, OR-ed into the working set.
 *
 * Defines (WISE paper section 3 "attention support", section 6.1, and the
 * temporal union of appendix B "WISE configuration"): for every (bh, q) the
 * admissible blocks b <= q are ranked by mass[bh][q][b], descending, ties to
 * the lower block index; the support is the shortest prefix whose cumulative
 * mass is >= eta.  If eta >= 1, or no prefix reaches eta, every admissible
 * block is kept.  Masses are clamped to [0, 1] (NaN counts as 0); cumulative sums
 * are exact sums of the masses rounded to multiples of 2^-21, and a prefix reaches
 * eta when that sum is at least ceil(eta * 2^21) * 2^-21 (so the result does not
 * depend on summation order).
 *
 * mass       : fp32 [B, H, nq, nq] (entries b > q are not read).
 * union_bits : uint32 [B, H, nq, W], W = ceil(nq / 32), in/out.  Bit (b % 32)
 *              of word b / 32 of row (bh, q) is set for every selected block
 *              (bit-or accumulate).  The caller zeroes it before the first
 *              window step.
 * step_bits  : uint32 [B, H, nq, W] output of this step's support alone, or NULL.
 * eta        : in (0, 1] ... values > 1 behave like 1.
 * Errors     : WISE_ERR_ARG (NULL mass/union_bits, eta <= 0 or NaN), WISE_ERR_SHAPE,
 *              WISE_ERR_CUDA.
 */
int wise_select_union(const float* mass, uint32_t* union_bits, uint32_t* step_bits, float eta,
                      wise_shape_t shape, void* stream);

/*
 * Block-size variant of wise_select_union: the support is chosen on blocks of
 * `block` tokens and run as exact 32 x 32 subtiles (WISE paper appendix C.6,
 * "Block-Size Tradeoff").
 *
 * Defines: with F = block / 32, the mass of coarse block B for coarse query
 * block Q is the block mass at block size 32F, R_QB = (1/F) sum over the F fine
 * query blocks q of Q and the fine key blocks b <= q of B of mass[bh][q][b]
 * (the block-mass equation of section 5.1 pooled exactly).  The coarse support
 * is chosen as in wise_select_union (rank descending, ties to the lower coarse
 * index, shortest prefix with cumulative mass >= eta, sums as there).  Fine row
 * q = Q F + a then keeps fine block b iff coarse block b / F is kept and b <= q.
 *
 * mass, union_bits, step_bits, eta : as for wise_select_union; the bit masks
 *              keep the fine [B, H, nq, W] layout, so wise_build_schedule and
 *              wise_sparse_attn consume them unchanged.
 * block      : 32, 64 or 128 tokens; 32 is exactly wise_select_union.
 * Errors     : WISE_ERR_ARG (as wise_select_union, or another block size),
 *              WISE_ERR_SHAPE (seqlen not a multiple of block, or as
 *              wise_select_union), WISE_ERR_CUDA.
 */
int wise_select_union_blocks(const float* mass, uint32_t* union_bits, uint32_t* step_bits,
                             float eta, int32_t block, wise_shape_t shape, void* stream);

/*
 * Block size 16 (WISE paper appendix C.6, "Block-Size Tradeoff": B in {16, 32, 64,
 * 128}).  Selection runs on 16-token blocks; execution keeps 32 x 32 tiles, each
 * carrying which of its four 16 x 16 sub-blocks are kept, so exactly the 16-token
 * support is attended.  With n16 = seqlen / 16 and W16 = ceil(n16 / 32):
 *
 * wise_block_mass_b16: r[bh][q][b] = (1/16) sum over the 16 rows i of block q and the
 *   keys j <= i of block b of exp(s_ij * scale - lse_i) (the block-mass equation of
 *   section 5.1 at B = 16), for b <= q; entries b > q within the diagonal 32 x 32
 *   block are written 0, the rest of b > q is not written.  QK^T is recomputed;
 *   lse is the natural-log lse of wise_full_attn_mass.
 *   q, k : bf16 [B, H, n, d] (k: [B, kv_heads, n, d]), 16-byte aligned;
 *   lse  : fp32 [B, H, n];  mass16 : fp32 [B, H, n16, n16] output.
 * wise_full_attn_mass_b16: wise_full_attn_mass (o, lse) plus the same mass16 in one pass:
 *   the attention kernel records every row's log-sum-exp over each 16-key half block in
 *   `workspace` (wise_mass_b16_workspace_bytes(shape) bytes, 16-byte aligned) and a
 *   light kernel averages 2^(blse - lse) over each block's 16 rows; no QK^T recompute.
 *   All pointers required.
 * wise_select_union_b16: wise_select_union over 16-token blocks: mass16 as above,
 *   union16 / step16 uint32 [B, H, n16, W16] (same bit layout, OR-accumulated /
 *   overwritten), same ranking, cut and eta rules.
 * wise_build_schedule_b16: the CSR schedule over 32-token query and key blocks
 *   (row_offsets [B*H*nq + 1], col_idx ascending per row, as wise_build_schedule)
 *   listing key block b for query block q when any 16-block pair (2q + a, 2b + c),
 *   a, c in {0, 1}, with 2b + c <= 2q + a is set in union16; sub[e] (uint8) holds
 *   those four bits of entry e at bit 2a + c.  Workspace: device memory of
 *   wise_schedule_b16_workspace_bytes(shape); capacity, nnz_out and errors as for
 *   wise_build_schedule.
 * wise_sparse_attn_b16: wise_sparse_attn where row i (16-row a = (i % 32) / 16)
 *   attends key j of a listed block only if bit 2a + (j % 32) / 16 of the entry's
 *   sub byte is set (and j <= i).  A row left with no key gets O = 0, lse = -inf.
 *   An entry whose sub byte has no bit set is skipped.
 * Errors: WISE_ERR_ARG (NULL pointers, eta <= 0, negative sizes), WISE_ERR_ALIGN,
 *   WISE_ERR_SHAPE, WISE_ERR_WORKSPACE, WISE_ERR_CAPACITY, WISE_ERR_CUDA.
 */
int wise_block_mass_b16(const void* q, const void* k, const float* lse, float* mass16,
                        wise_shape_t shape, void* stream);
int wise_full_attn_mass_b16(const void* q, const void* k, const void* v, void* o, float* lse,
                            float* mass16, void* workspace, size_t workspace_bytes,
                            wise_shape_t shape, void* stream);
/* Workspace bytes of wise_full_attn_mass_b16: B * H * (2 nq) * n * 4. */
size_t wise_mass_b16_workspace_bytes(wise_shape_t shape);
int wise_select_union_b16(const float* mass16, uint32_t* union16, uint32_t* step16, float eta,
                          wise_shape_t shape, void* stream);
size_t wise_schedule_b16_workspace_bytes(wise_shape_t shape);
int wise_build_schedule_b16(const uint32_t* union16, int32_t* row_offsets, int32_t* col_idx,
                            uint8_t* sub, int64_t col_capacity, int64_t* nnz_out,
                            void* workspace, size_t workspace_bytes, wise_shape_t shape,
                            void* stream);
int wise_sparse_attn_b16(const void* q, const void* k, const void* v, void* o,
                         const int32_t* row_offsets, const int32_t* col_idx, const uint8_t* sub,
                         int64_t col_count, float* lse, wise_shape_t shape, void* stream);

/*
 * Selection-only controls (WISE paper appendix B, "Intervention controls").  Both
 * take the block masses of recurrent step 1 and a reference working set (normally
 * the WISE union after step t_d) and write a support of the same layout, which
 * wise_build_schedule turns into a schedule like any other.  (The third control,
 * Static-95, is wise_select_union on the step-1 masses into a zeroed mask.)
 *
 * wise_select_size_matched (SizeMatched): row (bh, q) keeps the K admissible blocks
 *   of largest mass, K = the number of set admissible bits of the reference row;
 *   ties go to the lower block index.  K = 0 gives an empty row.
 * wise_select_mass_matched (MassMatched): m = the sum of the masses of the
 *   reference row's set admissible blocks; the row keeps the cumulative-eta support
 *   at eta = m (rank descending, ties to the lower index, shortest prefix with
 *   cumulative mass >= m; m >= 1 keeps every admissible block).  m and the prefix
 *   sums are the exact fixed-point sums of wise_select_union, so a reference row that
 *   is itself a ranking prefix is reproduced exactly.  m = 0 gives an empty row.
 *
 * mass     : fp32 [B, H, nq, nq] (entries b > q are not read).
 * ref_bits : uint32 [B, H, nq, W] (bits b > q are ignored).
 * out_bits : uint32 [B, H, nq, W] output (overwritten, not OR-ed); must not alias
 *            ref_bits.
 * Errors   : WISE_ERR_ARG (NULL pointer, aliasing), WISE_ERR_SHAPE, WISE_ERR_CUDA.
 */
int wise_select_size_matched(const float* mass, const uint32_t* ref_bits, uint32_t* out_bits,
                             wise_shape_t shape, void* stream);
int wise_select_mass_matched(const float* mass, const uint32_t* ref_bits, uint32_t* out_bits,
                             wise_shape_t shape, void* stream);

/*
 * Retained attention mass of a support (WISE paper appendix B, "Evaluation
 * metrics": the fraction of the unrestricted attention mass of a step that falls
 * inside the frozen support).  retained[bh][q] = sum of mass[bh][q][b] over the
 * admissible blocks b <= q whose bit is set, in fp32; with the block masses of a
 * late step and the frozen working set this is the retained future mass of query
 * block q (the mean over q is the per-token average).
 *
 * mass     : fp32 [B, H, nq, nq];  bits : uint32 [B, H, nq, W];
 * retained : fp32 [B, H, nq] output.
 * Errors   : WISE_ERR_ARG (NULL pointer), WISE_ERR_SHAPE, WISE_ERR_CUDA.
 */
int wise_support_mass(const float* mass, const uint32_t* bits, float* retained,
                      wise_shape_t shape, void* stream);

/* Workspace bytes wise_build_schedule needs for this shape (device memory). */
size_t wise_schedule_workspace_bytes(wise_shape_t shape);

/* Largest possible schedule size: BH * nq * (nq + 1) / 2 entries. */
int64_t wise_schedule_max_nnz(wise_shape_t shape);

/*
 * Compact the working set into the GPU-resident CSR schedule (WISE paper,
 * appendix B "Sparse-kernel implementation": row offsets plus active block
 * indices per recurrent block, head and query block).
 *
 * union_bits  : uint32 [B, H, nq, W] as produced by wise_select_union.  Bits
 *               for blocks b > q are ignored.
 * row_offsets : int32 [B*H*nq + 1] output; row r = bh * nq + q spans
 *               col_idx[row_offsets[r] .. row_offsets[r+1]).
 * col_idx     : int32 [col_capacity] output, key-block indices ascending per row.
 * nnz_out     : HOST int64 pointer or NULL.  If non-NULL the call synchronises
 *               `stream`, stores the entry count and returns WISE_ERR_CAPACITY
 *               if it exceeds col_capacity (col_idx then holds the first
 *               col_capacity entries).  If NULL, col_capacity must be at least
 *               wise_schedule_max_nnz(shape).
 * workspace   : device scratch of at least wise_schedule_workspace_bytes(shape).
 * Errors      : WISE_ERR_ARG, WISE_ERR_SHAPE, WISE_ERR_WORKSPACE, WISE_ERR_CAPACITY,
 *               WISE_ERR_CUDA.
 */
int wise_build_schedule(const uint32_t* union_bits, int32_t* row_offsets, int32_t* col_idx,
                        int64_t col_capacity, int64_t* nnz_out, void* workspace,
                        size_t workspace_bytes, wise_shape_t shape, void* stream);

/*
 * wise_build_schedule without a caller-provided workspace.
 *
 * The WISE paper has no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory, e.g. code embedded in a host framework
 * that owns every device allocation through its own pool, or a latency-bound
 * serving loop where cudaMalloc (which can synchronise the device) is not
 * allowed after start-up.  It computes exactly what wise_build_schedule
 * computes, with the same arguments minus the workspace, and allocates
 * nothing: its scan scratch is a fixed 16 KiB device array inside the
 * library, which every GPU that loads the library holds until the process
 * exits.
 *
 * Limit      : batch * heads * seqlen / 32 <= 1,048,576 schedule rows; larger
 *              shapes return WISE_ERR_WORKSPACE (use wise_build_schedule).
 * Set-up     : the first call on each device looks up the array's device
 *              address (with that device current) and keeps it with the id of
 *              the current CUDA context; a call in another context (a second
 *              context on the device, or the primary context after
 *              cudaDeviceReset) looks it up again.  Make the first call in each
 *              context before any stream capture.
 * Sharing    : all calls on a device use the same array and it keeps the last
 *              call's contents (nothing in it needs clearing: every entry read
 *              is written first by the same call).  Calls whose kernels overlap
 *              on the GPU, e.g. on unordered streams, race on it.
 * Errors     : as wise_build_schedule, with WISE_ERR_WORKSPACE for the limit.
 */
int wise_build_schedule_static(const uint32_t* union_bits, int32_t* row_offsets, int32_t* col_idx,
                               int64_t col_capacity, int64_t* nnz_out, wise_shape_t shape,
                               void* stream);

/*
 * Late-step block-sparse causal attention over a CSR schedule.
 *
 * Defines (WISE paper section 5.2, reuse mask R, and section 7.4): the dense
 * attention of wise_full_attn_mass restricted to keys j with j <= i and
 * block(j) in the schedule row of block(i); absent blocks are skipped, not
 * masked.  Q, K, V are this step's fresh values.
 *
 * row_offsets, col_idx : the schedule (see wise_build_schedule); each row's
 *               indices must be ascending and <= its query block.  Entries
 *               outside [0, col_count) or violating that order are skipped and
 *               flag WISE_STATUS_BAD_SCHEDULE; a row whose offsets are not
 *               ascending within [0, col_count] is treated as empty and flagged.
 *               Neither causes an out-of-range access.
 * col_count   : number of valid entries in col_idx (row_offsets[B*H*nq]).
 * lse         : fp32 [B, H, n] output or NULL.
 * A row whose schedule row is empty gets O = 0 and lse = -inf.
 * Errors      : WISE_ERR_ARG, WISE_ERR_SHAPE, WISE_ERR_ALIGN, WISE_ERR_CUDA.
 */
int wise_sparse_attn(const void* q, const void* k, const void* v, void* o,
                     const int32_t* row_offsets, const int32_t* col_idx, int64_t col_count,
                     float* lse, wise_shape_t shape, void* stream);

/*
 * Diagnostic (no counterpart in the WISE paper): exercise the bounded pipeline
 * wait of the kernels.  Launches one warp that waits, with the same bounded wait
 * the attention kernels use, on an mbarrier phase nothing completes; after
 * limit_ns nanoseconds the wait gives up, sets WISE_STATUS_TIMEOUT in the device
 * status word and the kernel returns (the context stays usable).  limit_ns must
 * be in (0, 10 s].  Errors: WISE_ERR_ARG, WISE_ERR_CUDA.
 */
int wise_diag_wait_timeout(uint64_t limit_ns, void* stream);

/*
 * Read (and optionally clear) the device status word of the current device.
 * Synchronises the device.  *status_out receives WISE_STATUS_* bits.
 */
int wise_device_status(uint32_t* status_out, int clear);

/* Message of the last error returned on this thread ("" if none). */
const char* wise_last_error(void);

/* Library version string. */
const char* wise_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WISE_H_ */
