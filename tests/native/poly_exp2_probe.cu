// Applies the prefill softmax's FMA-pipe exponential (pkv::tc::poly_exp2) elementwise, so a
// GPU test can compare it with CUDA's exp2f; compiled by tests/test_poly_exp2.py on the GPU machine.
#include <cuda_runtime.h>

#include "tcgen05_common.cuh"

__global__ void poly_exp2_probe_kernel(const float* x, float* y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = pkv::tc::poly_exp2(x[i]);
}

extern "C" int poly_exp2_probe(const float* x, float* y, int n, void* stream) {
  if (n <= 0) return 0;
  poly_exp2_probe_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return static_cast<int>(cudaGetLastError());
}
