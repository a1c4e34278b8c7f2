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

}  // namespace pkv
