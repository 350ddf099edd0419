// diag.cu -- diagnostic entry points (no counterpart in the WISE paper).

#include <cuda_runtime.h>

#include "sm100.cuh"
#include "wise.h"
#include "wise_internal.h"

namespace wise {

// One warp waits, through the same bounded mbar_wait the attention kernels use,
// on an mbarrier phase that nothing completes.  The wait must give up after
// limit_ns, record kStatusTimeout and let the kernel return.
__global__ void diag_wait_timeout_kernel(unsigned long long limit_ns, unsigned int* status) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait(smem_u32(&bar), 0, &abort_flag, status, limit_ns);
  __syncwarp();
}

}  // namespace wise

extern "C" int wise_diag_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 10000000000ull)
    return wise::record_error(WISE_ERR_ARG, "limit_ns must be in (0, 10 s]");
  unsigned int* st = nullptr;
  const int rc = wise::status_word(&st);
  if (rc) return rc;
  wise::diag_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, st);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return wise::record_error(WISE_ERR_CUDA, cudaGetErrorString(e));
  return wise::record_ok();
}
