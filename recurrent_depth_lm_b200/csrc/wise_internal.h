// wise_internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "wise.h"

namespace wise {

// kModeSparse16: block-sparse attention whose 32 x 32 blocks carry 16 x 16 sub-masks
// (block size 16).
enum { kModeDense = 0, kModeSparse = 1, kModeMass = 2, kModeSparse16 = 3 };

struct AttnParams {
  int BH;               // batch * heads
  int group;            // query heads per K/V head: K/V head of bh is bh / group
  int n;                // sequence length
  int nq;               // n / 32
  int num_tiles;        // BH * ceil(nq / 4)
  float scale_log2;     // softmax scale * log2(e)
  void* o;              // [BH, n, d] bf16 output (dense / sparse)
  float* lse;           // [BH, n] output (dense / sparse), nullable
  const float* lse_in;  // [BH, n] input (mass mode)
  float* mass;          // [BH, nq, nq] output (mass mode); [BH, 2nq, 2nq] when fine16
  int fine16;           // mass mode: block mass of 16-token blocks; dense mode with blse:
                        // one blse per 16-key half ([BH, 2nq, n])
  float* blse;          // [BH, nq, n] block log2-sum-exp side output (dense mode), nullable
  const int32_t* row_offsets;  // sparse mode
  const int32_t* col_idx;      // sparse mode
  long long col_count;         // sparse mode: valid entries of col_idx
  const uint8_t* sub;          // sparse16 mode: 16 x 16 sub-mask bits of each col_idx entry
  unsigned int* status;        // device status word
};

// On a launch-configuration failure specific to the kernel, *why gets a description.
cudaError_t launch_attention(int mode, int d, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, const AttnParams& p, int grid,
                             cudaStream_t stream, const char** why);
int attention_smem_bytes(int mode, int d);

// mass[bh][q][b] = (1/32) sum_{i in q} 2^(blse[bh][b][i] - lse[bh][i] * log2 e), b <= q
// Block mass from the recorded per-(row, key block) log-sum-exps.
cudaError_t launch_block_mass(const float* blse, const float* lse, float* mass, int BH, int n,
                              cudaStream_t stream);
// The same at 16-token blocks: blse16 is [BH, 2nq, n], mass16 [BH, 2nq, 2nq]; for b > q it
// writes the diagonal 32-block's entry (0) and nothing else.
cudaError_t launch_block_mass16(const float* blse16, const float* lse, float* mass16, int BH,
                                int n, cudaStream_t stream);

cudaError_t launch_select_union(const float* mass, uint32_t* union_bits, uint32_t* step_bits,
                                float eta, int BH, int nq, cudaStream_t stream);

// Selection on blocks of factor x 32 tokens (factor 1, 2 or 4; nq % factor == 0),
// written back as fine 32 x 32 masks in the [BH, nq, W] layout.
cudaError_t launch_select_union_blocks(const float* mass, uint32_t* union_bits,
                                       uint32_t* step_bits, float eta, int factor, int BH, int nq,
                                       cudaStream_t stream);

// Selection-only controls from a reference mask: kind 0 = SizeMatched (TopK, K = |ref row|),
// kind 1 = MassMatched (cumulative cut at the mass of the ref row).
cudaError_t launch_select_control(const float* mass, const uint32_t* ref_bits, uint32_t* out_bits,
                                  int kind, int BH, int nq, cudaStream_t stream);

// retained[bh * nq + q] = sum of mass over the set admissible bits of the row.
cudaError_t launch_support_mass(const float* mass, const uint32_t* bits, float* retained, int BH,
                                int nq, cudaStream_t stream);

// Block size 16: fold the [BH, 2nq, W16] 16-token masks into 32-token rows [BH, nq, W]
// (a 32-block is kept if any of its four 16-blocks is, causally), then the sub-mask of
// every schedule entry: bit 2a + c = 16-row 2q + a keeps 16-block 2b + c.
cudaError_t launch_fold16(const uint32_t* union16, uint32_t* bits32, int BH, int nq,
                          cudaStream_t stream);
cudaError_t launch_sub16(const uint32_t* union16, const int32_t* row_offsets,
                         const int32_t* col_idx, uint8_t* sub, long long capacity, int BH,
                         int nq, cudaStream_t stream);

size_t schedule_workspace_bytes(long long rows);
cudaError_t launch_build_schedule(const uint32_t* union_bits, int32_t* row_offsets,
                                  int32_t* col_idx, long long capacity, void* workspace,
                                  long long rows, int nq, cudaStream_t stream);

// Error recording and shape validation shared with entry points outside api.cu.
int record_error(int code, const char* msg);
int record_ok();
int validate_shape(const wise_shape_t& s);
// Device address of the current device's status word.
int status_word(unsigned int** out);
// Id of the calling thread's current CUDA context (unique for the life of the process;
// a reset primary context gets a new one); false if there is none or the driver lacks
// cuCtxGetId.
bool current_context_id(unsigned long long* id);

}  // namespace wise
