// launch.cuh - kernel launches with programmatic dependent launch (PDL, sm_90 and later).
//
// Every kernel of the layer is launched with the programmatic stream-serialisation
// attribute: the next kernel on the stream may be scheduled as soon as every CTA of the
// running one has executed pdl_launch_dependents(), so its set-up (barrier initialisation,
// TMEM allocation, tensor-map prefetch) overlaps the tail of its predecessor. The contract
// each kernel keeps:
//   * before pdl_wait() it touches no global memory except kernel parameters and
//     tensor maps (no reads of anything a kernel writes, no writes at all);
//   * every thread that reads or writes global memory has executed pdl_wait() first, and
//     every CTA executes it before exiting (so a kernel never completes ahead of the one
//     it depends on, and completion stays transitive down the stream).
// pdl_wait() returns once all prerequisite grids have completed and their memory is
// visible; without the attribute (MOE_TUNE_PDL set to 0) it returns at once.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace moe {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// False when moe_set_tuning(MOE_TUNE_PDL, 0) is in effect.
bool pdl_enabled();

// kern<<<grid, block, smem, st>>>(args...) with the PDL attribute (and, for cluster > 1,
// a cluster of that many CTAs along x).
template <typename... P, typename... A>
cudaError_t launch_kernel(void (*kern)(P...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, unsigned cluster, A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  ++n;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

}  // namespace moe
