// launch.cuh — every kernel of the library is launched through launch_k():
// cudaLaunchKernelEx with programmatic dependent launch enabled (and, for the
// skinny GEMMs, a 1 x 1 x cz cluster).  Each kernel calls pdl_wait() before its
// first access to global memory, and most call pdl_launch_dependents() right
// after it, so the next kernel's CTAs can be placed and run their prologue
// (barrier init, TMEM allocation, tensor-map prefetch) while this one runs;
// stream order for memory is unchanged.  The kernels of gemm.cuh and
// gemm_pair.cuh do not trigger early (see gemm.cuh): the grid after them starts
// when they have finished, except that s·X·A lets the small-M forward start early.
// They are also launched without the programmatic attribute (launch_k_ordered),
// the small-M forward with it.
// Because a kernel triggers its dependents only after its own wait returned,
// every grid before its predecessor is complete when a dependent starts: a
// dependent that reads some inputs before its own wait may rely on that (it must
// still wait before reading its predecessor's output).
#pragma once
#include <atomic>
#include <cstdint>
#include <utility>
#include <cuda_runtime.h>
#include "internal.h"

namespace qlora {

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device once.  The attribute belongs to the device's context, so `done` holds
// one bit per device (devices 64 and up set it on every call).  Two host threads
// that race here both set the same value, which is harmless.
inline cudaError_t smem_attr_once(const void *kern, int bytes, std::atomic<uint64_t> &done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_k_pdl(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                         unsigned cz, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  ++n;
  if (cz > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = 1;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = cz;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  count_launches(1);
  // consume the launch's error state either way, so that a failed launch is not
  // reported again by the next one
  const cudaError_t last = cudaGetLastError();
  return e != cudaSuccess ? e : last;
}

// Programmatic dependent launch on: the kernel may start as soon as its predecessor
// triggers (it still waits for it before touching memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, unsigned cz,
                     Args &&...args) {
  return launch_k_pdl(true, kern, grid, block, smem, st, cz, std::forward<Args>(args)...);
}

// Plain stream order: the kernel starts when its predecessor has finished.  Used for
// the dequant and adapter GEMMs (gemm.cuh, gemm_pair.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_k_ordered(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             unsigned cz, Args &&...args) {
  return launch_k_pdl(false, kern, grid, block, smem, st, cz, std::forward<Args>(args)...);
}

}  // namespace qlora
