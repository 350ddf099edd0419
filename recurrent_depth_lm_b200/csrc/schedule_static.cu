// schedule_static.cu -- wise_build_schedule_static: the CSR schedule build of
// wise_build_schedule with its scratch memory held in a fixed device array
// inside the library, for callers that cannot allocate device memory.
//
// The scan scratch (one int per 256 schedule rows) lives in g_sched_scratch, a
// file-scope __device__ array of kStaticScratchInts ints (16 KiB).  Every GPU
// that loads the library holds it until the process exits.  Host code cannot
// use the array's name as a device address, so the first call on each device
// looks the address up with cudaGetSymbolAddress (with that device current)
// and caches it with the id of the current CUDA context; a call made in another
// context (a second context on the device, or the primary context after a reset)
// looks it up again.  Make the first call in a context before any stream
// capture.  All calls on
// a device share the one array and it keeps the previous call's contents: the
// scan writes every entry it later reads, so nothing has to be cleared, but two
// calls whose kernels overlap on the GPU (different streams, no ordering) race
// on it.

#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "wise.h"
#include "wise_internal.h"

namespace {

constexpr long long kStaticScratchInts = 4096;      // 16 KiB
constexpr long long kRowsPerScratchInt = 256;       // schedule rows per block sum
constexpr long long kStaticMaxRows = kStaticScratchInts * kRowsPerScratchInt;  // 1,048,576

static __device__ __align__(256) int g_sched_scratch[kStaticScratchInts];

constexpr int kMaxDevices = 64;
struct ScratchAddr {
  int* ptr = nullptr;
  unsigned long long ctx = 0;   // id of the context ptr belongs to
};
ScratchAddr g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of g_sched_scratch in the current context (set up once per device and
// context; without a context id, e.g. on a driver that lacks cuCtxGetId, on every call).
int scratch_on_current_device(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return wise::record_error(WISE_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return wise::record_error(WISE_ERR_CUDA, "device index out of range");
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchAddr& sa = g_scratch[dev];
  unsigned long long ctx = 0;
  const bool have_ctx = wise::current_context_id(&ctx);
  if (sa.ptr == nullptr || !have_ctx || sa.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_sched_scratch);   // creates the context if needed
    if (e != cudaSuccess) {
      char msg[256];
      snprintf(msg, sizeof(msg), "cudaGetSymbolAddress(schedule scratch): %s",
               cudaGetErrorString(e));
      return wise::record_error(WISE_ERR_CUDA, msg);
    }
    *out = static_cast<int*>(p);
    sa.ptr = wise::current_context_id(&sa.ctx) ? *out : nullptr;
    return WISE_OK;
  }
  *out = sa.ptr;
  return WISE_OK;
}

}  // namespace

extern "C" int wise_build_schedule_static(const uint32_t* union_bits, int32_t* row_offsets,
                                          int32_t* col_idx, int64_t col_capacity,
                                          int64_t* nnz_out, wise_shape_t shape, void* stream) {
  int rc = wise::validate_shape(shape);
  if (rc) return rc;
  if (!union_bits || !row_offsets || !col_idx)
    return wise::record_error(WISE_ERR_ARG,
                              "union_bits, row_offsets and col_idx must be non-NULL");
  if (col_capacity < 0) return wise::record_error(WISE_ERR_ARG, "col_capacity must be >= 0");
  const long long nq = shape.seqlen / 32;
  const long long rows = (long long)shape.batch * shape.heads * nq;
  if (rows > kStaticMaxRows) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "schedule has %lld rows (batch*heads*seqlen/32); the fixed scratch of this entry "
             "point covers at most %lld rows - use wise_build_schedule with a workspace",
             rows, kStaticMaxRows);
    return wise::record_error(WISE_ERR_WORKSPACE, msg);
  }
  const long long max_nnz = rows * (nq + 1) / 2;
  if (max_nnz > 0x7fffffffll)
    return wise::record_error(WISE_ERR_SHAPE, "schedule may exceed 2^31 entries");
  if (!nnz_out && col_capacity < max_nnz)
    return wise::record_error(WISE_ERR_CAPACITY,
                              "col_capacity below the worst case; pass nnz_out to check the "
                              "exact size");
  int* scratch = nullptr;
  rc = scratch_on_current_device(&scratch);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = wise::launch_build_schedule(union_bits, row_offsets, col_idx, col_capacity,
                                              scratch, rows, (int)nq, st);
  if (e != cudaSuccess) return wise::record_error(WISE_ERR_CUDA, cudaGetErrorString(e));
  if (nnz_out) {
    int32_t nnz = 0;
    e = cudaMemcpyAsync(&nnz, row_offsets + rows, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return wise::record_error(WISE_ERR_CUDA, cudaGetErrorString(e));
    *nnz_out = nnz;
    if (nnz > col_capacity)
      return wise::record_error(WISE_ERR_CAPACITY, "schedule larger than col_capacity");
  }
  return wise::record_ok();
}
