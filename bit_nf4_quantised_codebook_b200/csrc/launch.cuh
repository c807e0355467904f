// launch.cuh — every kernel of the library is launched through launch_k():
// cudaLaunchKernelEx with programmatic dependent launch enabled (and, for the
// skinny GEMMs, a 1 x 1 x cz cluster).  Each kernel calls pdl_wait() before its
// first access to global memory and pdl_launch_dependents() right after it, so
// the next kernel's CTAs can be placed and run their prologue (barrier init,
// TMEM allocation, tensor-map prefetch) while this one runs; stream order for
// memory is unchanged.  Because a kernel triggers its dependents only after its
// own wait returned, every grid before its predecessor is complete when a
// dependent starts: a dependent that reads some inputs before its own wait may
// rely on that (it must still wait before reading its predecessor's output).
#pragma once
#include <utility>
#include <cuda_runtime.h>
#include "internal.h"

namespace qlora {

template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, unsigned cz,
                     Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
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
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace qlora
