// Self-test of the bounded waits every kernel of the library uses: a single
// CTA waits on an mbarrier that nothing ever arrives on.  The wait must give
// up after `timeout_ns`, record ERR_WAIT_TIMEOUT in the device error word and
// return, leaving the CUDA context usable (no trap, no hang).
#include <cuda_runtime.h>

#include <atomic>

#include "cp_attn.h"
#include "sm100_ptx.cuh"

namespace cp {
std::atomic<uint64_t>& launch_counter();
cudaError_t attn_err_word(uint32_t** dev_ptr);
void set_error_message(const char* msg);

__global__ void wait_timeout_kernel(uint32_t* err, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // phase 0 never completes: nobody arrives
  mbar_wait_warp(smem_addr(&bar), 0, &abort_flag, err, timeout_ns);
}
}  // namespace cp

extern "C" cp_status cp_selftest_wait_timeout(uint64_t timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) {
    cp::set_error_message("cp_selftest_wait_timeout: timeout must be in (0, 10 s]");
    return CP_ERR_INVALID_ARG;
  }
  uint32_t* err = nullptr;
  cudaError_t e = cp::attn_err_word(&err);
  if (e != cudaSuccess) {
    cp::set_error_message("cp_selftest_wait_timeout: error word unavailable");
    return CP_ERR_CUDA;
  }
  cp::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, timeout_ns);
  cp::launch_counter()++;
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    cp::set_error_message(cudaGetErrorString(e));
    return CP_ERR_CUDA;
  }
  return CP_OK;
}
