// Host-side launch of the path's kernels.
#pragma once

#include <cuda_runtime.h>

#include <utility>

namespace hinm {

// Launches kernel<<<grid, block, smem, s>>>(args...) with programmatic stream serialization
// allowed: the launch is processed while the previous kernel of the stream finishes, instead
// of after its completion has been signalled (a capture turns it into a programmatic graph
// edge).  Every kernel launched this way begins with ptx::enter_dependent(), whose wait
// keeps all its memory accesses after the previous kernels' completion.  Measured on B200,
// the five calls launched one by one: HiNM up-projection 486 -> 470 us, pure 2:4 271 ->
// 258 us, decode 441 -> 430 us; a replayed CUDA graph of the same calls is unchanged.  The
// arguments are converted to the kernel's parameter types.  extra (optional) is one more
// launch attribute (a cluster shape).
template <typename... Params, typename... Args>
cudaError_t launch_kernel(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, const cudaLaunchAttribute* extra, Args&&... args) {
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  unsigned n = 1;
  if (extra) attr[n++] = *extra;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace hinm
