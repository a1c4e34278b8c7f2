// Host-side launch set-up shared by the kernel launchers.
#pragma once

#include <cuda_runtime.h>

#include "per_device.h"

namespace pkv {

// Writes the current device to *dev and raises `kernel`'s dynamic shared-memory limit to
// `smem` bytes the first time it launches on that device (the limit belongs to each device's
// context).  Returns 0 or a cudaError_t value.
template <class Kernel>
inline int set_smem_limit_once(PerDevice<int>& setup, Kernel kernel, int smem, int* dev) {
  const cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return static_cast<int>(e);
  return setup.get(
      *dev,
      [&](int&) {
        return static_cast<int>(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
      },
      nullptr, static_cast<int>(cudaErrorInvalidDevice));
}

// Launches `kernel` with programmatic stream serialization: it may be scheduled (and run
// up to its griddep_wait()) while the previous kernel of `stream` is still running, which
// hides the launch gap between the kernels of one call.  The kernel must call griddep_wait()
// in every thread before it reads the previous kernel's output or returns.
template <typename... KernelParams, typename... Args>
inline cudaError_t launch_after_previous(void (*kernel)(KernelParams...), dim3 grid, dim3 block, size_t smem,
                                         cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace pkv
