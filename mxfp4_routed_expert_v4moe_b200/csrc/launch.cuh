// Kernel launch wrapper: every kernel of the library is launched through
// launch_kernel(), which counts launches and, when kernel timing is switched
// on (v4moe_profile_enable), brackets the launch with CUDA events recorded on
// the launch stream. Optional programmatic dependent launch (PDL) lets a
// kernel start its prologue while the previous one drains.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace v4moe {

// Profiler hooks (profile.cu). prof_begin returns an opaque slot or -1.
bool prof_enabled();
int prof_begin(const char* name, cudaStream_t st);
void prof_end(int slot, cudaStream_t st);
void count_launch();

// `cluster` > 0 launches thread-block clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel_cl(const char* name, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, bool pdl, int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  const bool prof = prof_enabled();
  if (pdl && !prof) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = unsigned(cluster);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = n ? attr : nullptr;
  cfg.numAttrs = n;
  const int slot = prof ? prof_begin(name, st) : -1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (slot >= 0) prof_end(slot, st);
  count_launch();
  return e;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(const char* name, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t st, bool pdl, Args&&... args) {
  return launch_kernel_cl(name, kern, grid, block, smem, st, pdl, 0, std::forward<Args>(args)...);
}

// Raise the dynamic shared memory limit of a kernel (cheap; done per launch so
// that every device the process uses gets it).
template <typename K>
inline void set_smem(K* kern, size_t bytes) {
  if (bytes > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
}

}  // namespace v4moe
