// Programmatic dependent launch. A kernel launched by launch_k may start while the kernel before
// it in the stream is still finishing: its CTAs take SMs as they free up, run their set-up
// (barrier init, TMEM allocation, descriptor prefetch), and wait in pdl_wait() until that kernel has
// completed and its memory operations are visible. Every kernel launched this way calls pdl_wait()
// before it touches global memory, and pdl_trigger() so that the next kernel may be scheduled
// once all of its own CTAs are running. Without the launch attribute both are no-ops. The
// environment variable LST_PDL=0 launches everything the plain way.
#pragma once

#include <cstdlib>
#include <cstring>
#include <utility>

#include <cuda_runtime.h>

namespace lst {

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

inline bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("LST_PDL");
    return !(e && std::strcmp(e, "0") == 0);
  }();
  return on;
}

// kernel<<<grid, block, smem, s>>>(args...) with programmatic stream serialization, and a thread-block
// cluster of cluster_x CTAs along x when cluster_x > 0.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                            unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  unsigned n = 0;
  if (pdl_enabled()) {
    at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 0) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = cluster_x;
    at[n].val.clusterDim.y = 1;
    at[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace lst
