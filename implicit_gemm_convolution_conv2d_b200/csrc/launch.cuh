// launch.cuh -- host-side kernel launch with programmatic stream serialization.
//
// Every kernel of this library lets the next launch on its stream start once
// its own setup (barrier init, tensor-memory allocation, tensor-map prefetch)
// is done, and waits for the previous grid on the stream to complete, with its
// writes visible, before its first access to global memory (ptx::pdl_* at the
// end of each kernel's setup).  Launched with the attribute below, a kernel's
// launch and setup then overlap the last CTAs of the kernel before it; the
// results are those of plain stream order.
#pragma once

#include <cuda_runtime.h>

namespace convfwd {

// `cluster` > 1 launches clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = static_cast<unsigned>(n);
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Adds programmatic stream serialization to a launch configuration that
// already holds cfg.numAttrs attributes in `attr` (room for one more).
inline void add_pdl(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attr) {
  attr[cfg.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[cfg.numAttrs].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  ++cfg.numAttrs;
}

}  // namespace convfwd
