// Cache writes of the decode step: reshape_and_cache (scatter new tokens' K/V into
// the block pool through their slots) and copy_blocks (copy-on-write block copies).
//
// Outcome School vLLM explainer, "LLM serving的基本流程与KV缓存": each decoded token
// adds one K/V pair that stays in GPU memory until the request ends; the
// intelliparadigm article §2.2: growth needs only a new page and a table update.
// Both kernels are plain 16-byte vector copies: bit-exact, HBM-bound, and tiny next
// to the attention read that follows them.
#include <cuda_runtime.h>

#include <algorithm>

#include "device_common.cuh"
#include "pkv_internal.h"

namespace pkv {

// One thread moves one 16-byte chunk of one (token, kv head) row, for K and for V.
// Consecutive threads cover consecutive chunks of a row, so both the source row
// and the destination row (contiguous inside the (block, head) tile) are coalesced.
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(const uint4* __restrict__ key,
                                                                const uint4* __restrict__ value,
                                                                uint4* __restrict__ key_cache,
                                                                uint4* __restrict__ value_cache,
                                                                const int64_t* __restrict__ slot_mapping,
                                                                int64_t total_chunks, int chunks_per_row,
                                                                int num_kv_heads, int block_size,
                                                                int64_t num_slots, int32_t* status) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total_chunks; i += stride) {
    const int c = static_cast<int>(i % chunks_per_row);
    const int64_t row = i / chunks_per_row;              // token * Hkv + head
    const int h = static_cast<int>(row % num_kv_heads);
    const int64_t t = row / num_kv_heads;
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (c == 0 && h == 0) set_status(status, PKV_DEV_BAD_SLOT);
      continue;
    }
    const int64_t block = slot / block_size;
    const int64_t r = slot - block * block_size;
    const int64_t dst = ((block * num_kv_heads + h) * block_size + r) * chunks_per_row + c;
    key_cache[dst] = key[i];
    value_cache[dst] = value[i];
  }
}

constexpr int kMaxLayersPerLaunch = 64;

struct CopyBlocksLayers {
  uint4* key[kMaxLayersPerLaunch];
  uint4* value[kMaxLayersPerLaunch];
};

// grid = (pairs, layers, 2 for K/V); each CTA copies one block of one pool.
__global__ void __launch_bounds__(256) copy_blocks_kernel(const __grid_constant__ CopyBlocksLayers layers,
                                                          const int64_t* __restrict__ block_mapping,
                                                          int num_blocks, int64_t chunks_per_block,
                                                          int32_t* status) {
  const int64_t src = block_mapping[2 * blockIdx.x];
  const int64_t dst = block_mapping[2 * blockIdx.x + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) set_status(status, PKV_DEV_BAD_PAIR);
    return;
  }
  uint4* pool = blockIdx.z == 0 ? layers.key[blockIdx.y] : layers.value[blockIdx.y];
  const uint4* s = pool + src * chunks_per_block;
  uint4* d = pool + dst * chunks_per_block;
  for (int64_t i = threadIdx.x; i < chunks_per_block; i += blockDim.x) d[i] = s[i];
}

static int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return PKV_OK;
}

static int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace pkv

using namespace pkv;

extern "C" int pkv_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                                     const int64_t* slot_mapping, int num_tokens, int num_blocks,
                                     int num_kv_heads, int head_dim, int block_size, int32_t* status,
                                     pkv_stream_t stream) {
  clear_error();
  if (num_tokens < 0 || num_blocks <= 0 || num_kv_heads <= 0)
    return set_error(PKV_ERR_INVALID, "reshape_and_cache: bad sizes");
  if (head_dim != 64 && head_dim != 128)
    return set_error(PKV_ERR_UNSUPPORTED, "reshape_and_cache: head_dim %d not in {64,128}", head_dim);
  if (block_size != 16 && block_size != 32)
    return set_error(PKV_ERR_UNSUPPORTED, "reshape_and_cache: block_size %d not in {16,32}", block_size);
  if (num_tokens == 0) return PKV_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping)
    return set_error(PKV_ERR_INVALID, "reshape_and_cache: null pointer");
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
    return set_error(PKV_ERR_INVALID, "reshape_and_cache: tensors must be 16-byte aligned");
  const int chunks_per_row = head_dim * 2 / 16;
  const int64_t total = static_cast<int64_t>(num_tokens) * num_kv_heads * chunks_per_row;
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int blocks = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(sm_count()) * 8));
  reshape_and_cache_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(key), static_cast<const uint4*>(value), static_cast<uint4*>(key_cache),
      static_cast<uint4*>(value_cache), slot_mapping, total, chunks_per_row, num_kv_heads, block_size,
      static_cast<int64_t>(num_blocks) * block_size, status);
  return check_launch("reshape_and_cache launch");
}

extern "C" int pkv_copy_blocks(void* const* key_caches, void* const* value_caches, int num_layers,
                               const int64_t* block_mapping, int num_pairs, int num_blocks,
                               int64_t block_elems, int32_t* status, pkv_stream_t stream) {
  clear_error();
  if (num_layers < 0 || num_pairs < 0 || num_blocks <= 0 || block_elems <= 0)
    return set_error(PKV_ERR_INVALID, "copy_blocks: bad sizes");
  if ((block_elems * 2) % 16 != 0)
    return set_error(PKV_ERR_INVALID, "copy_blocks: block bytes must be a multiple of 16");
  if (num_layers == 0 || num_pairs == 0) return PKV_OK;
  if (!key_caches || !value_caches || !block_mapping) return set_error(PKV_ERR_INVALID, "copy_blocks: null pointer");
  for (int l = 0; l < num_layers; ++l)
    if (!key_caches[l] || !value_caches[l] || !aligned16(key_caches[l]) || !aligned16(value_caches[l]))
      return set_error(PKV_ERR_INVALID, "copy_blocks: layer %d pool is null or not 16-byte aligned", l);
  const int64_t chunks = block_elems * 2 / 16;
  for (int l0 = 0; l0 < num_layers; l0 += kMaxLayersPerLaunch) {
    const int nl = std::min(kMaxLayersPerLaunch, num_layers - l0);
    CopyBlocksLayers layers{};
    for (int l = 0; l < nl; ++l) {
      layers.key[l] = static_cast<uint4*>(key_caches[l0 + l]);
      layers.value[l] = static_cast<uint4*>(value_caches[l0 + l]);
    }
    dim3 grid(num_pairs, nl, 2);
    copy_blocks_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(layers, block_mapping, num_blocks,
                                                                           chunks, status);
    int rc = check_launch("copy_blocks launch");
    if (rc != PKV_OK) return rc;
  }
  return PKV_OK;
}
