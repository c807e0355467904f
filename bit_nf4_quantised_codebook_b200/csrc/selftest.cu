// selftest.cu — exercises, on the device, the error path that every pipeline
// wait of the library takes when its bound runs out, without any fault: one
// CTA waits on an mbarrier that nothing ever arrives on, through the same
// bounded wait the GEMM and quantiser pipelines use.  The wait gives up after
// `timeout_ns`, raises the CTA's abort flag and records QLORA_DEVERR_TIMEOUT in
// *dev_err; the kernel then returns normally and the context stays usable.
#include <cstdint>
#include <cuda_runtime.h>
#include "internal.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace qlora {

__global__ void k_selftest_wait(unsigned long long timeout_ns, int *dev_err, int *gave_up) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival would complete phase 0; none ever comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait_bounded(&bar, 0, &abort_flag, dev_err, timeout_ns);
    if (gave_up) *gave_up = ok ? 0 : 1;
  }
}

cudaError_t launch_selftest_wait(unsigned long long timeout_ns, int *dev_err, int *gave_up, cudaStream_t st) {
  return launch_k(k_selftest_wait, dim3(1), dim3(32), 0, st, 1, timeout_ns, dev_err, gave_up);
}

}  // namespace qlora
