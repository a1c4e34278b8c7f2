// Read-only streaming of a device buffer: the HBM read bandwidth that the decode
// kernels' roofline is compared with, measured in the same run as them.
//
// Every thread keeps four 16-byte non-caching loads in flight over a grid-stride walk
// and folds the words with XOR, so the loads cannot be dropped and the result can be
// checked bit for bit; each CTA folds its warps and makes one atomicXor.
#include <cuda_runtime.h>

#include "device_common.cuh"
#include "pkv_internal.h"

namespace pkv {

constexpr int kStreamThreads = 512;

__device__ __forceinline__ uint4 load_nc(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(kStreamThreads) stream_read_kernel(const uint4* __restrict__ src, int64_t n,
                                                                      uint32_t* __restrict__ sink) {
  __shared__ uint32_t warp_x[kStreamThreads / 32];
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  uint32_t x = 0;
  for (; i + 3 * stride < n; i += 4 * stride) {
    const uint4 a = load_nc(src + i), b = load_nc(src + i + stride);
    const uint4 c = load_nc(src + i + 2 * stride), d = load_nc(src + i + 3 * stride);
    x ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w ^ c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^ d.z ^ d.w;
  }
  for (; i < n; i += stride) {
    const uint4 a = load_nc(src + i);
    x ^= a.x ^ a.y ^ a.z ^ a.w;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x ^= __shfl_xor_sync(0xffffffffu, x, off);
  if ((threadIdx.x & 31) == 0) warp_x[threadIdx.x >> 5] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0;
    for (int w = 0; w < kStreamThreads / 32; ++w) b ^= warp_x[w];
    atomicXor(sink, b);
  }
}

}  // namespace pkv

using namespace pkv;

extern "C" int pkv_stream_read(const void* src, size_t bytes, uint32_t* sink, pkv_stream_t stream) {
  clear_error();
  if (bytes % 16 != 0) return set_error(PKV_ERR_INVALID, "stream_read: bytes must be a multiple of 16");
  if (bytes == 0) return PKV_OK;
  if (!src || !sink) return set_error(PKV_ERR_INVALID, "stream_read: null pointer");
  if (!aligned16(src) || (reinterpret_cast<uintptr_t>(sink) & 3u) != 0)
    return set_error(PKV_ERR_INVALID, "stream_read: src must be 16-byte and sink 4-byte aligned");
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t n = static_cast<int64_t>(bytes / 16);
  const int64_t want = (n + kStreamThreads - 1) / kStreamThreads;
  const int grid = static_cast<int>(want < 4LL * sms ? want : 4LL * sms);  // 4 CTAs of 512 threads per SM
  stream_read_kernel<<<grid, kStreamThreads, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<const uint4*>(src),
                                                                                     n, sink);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "stream_read launch: %s", cudaGetErrorString(e));
  return PKV_OK;
}
