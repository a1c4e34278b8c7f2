// Cache writes of the decode step: reshape_and_cache (scatter new tokens' K/V into
// the block pool through their slots) and copy_blocks (copy-on-write block copies).
//
// Outcome School vLLM explainer, "LLM serving的基本流程与KV缓存": each decoded token
// adds one K/V pair that stays in GPU memory until the request ends; the
// intelliparadigm article §2.2: growth needs only a new page and a table update.
// Both kernels are plain 16-byte vector copies: bit-exact, HBM-bound, and tiny next
// to the attention read that follows them.
//
// Also here: the quantising write of an 8-bit (e4m3) pool (intelliparadigm article
// §4.2/§5: low-bit storage), and swap_blocks, the pool's overflow path to pinned
// host memory (§4.2 OOM错误: swap_space), as one kernel over every block pair.
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

// e4m3 quantisation of 16 values: x / scale, correctly rounded in fp32, then round
// to nearest even into e4m3 with saturation to +-448.
__device__ __forceinline__ uint32_t e4m3x4(float x0, float x1, float x2, float x3) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(x1), "f"(x0));  // first operand -> high byte
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(x3), "f"(x2));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

__device__ __forceinline__ uint4 quantize16(const uint4 a, const uint4 b, float s) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t r[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    r[i] = e4m3x4(__fdiv_rn(bf16lo(w[2 * i]), s), __fdiv_rn(bf16hi(w[2 * i]), s), __fdiv_rn(bf16lo(w[2 * i + 1]), s),
                  __fdiv_rn(bf16hi(w[2 * i + 1]), s));
  return make_uint4(r[0], r[1], r[2], r[3]);
}

// One thread writes one 16-byte chunk (16 codes) of one (token, kv head) row of K and V.
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(
    const uint4* __restrict__ key, const uint4* __restrict__ value, uint4* __restrict__ key_cache,
    uint4* __restrict__ value_cache, const int64_t* __restrict__ slot_mapping, const float* __restrict__ k_scale,
    const float* __restrict__ v_scale, int64_t total_chunks, int chunks_per_row, int num_kv_heads, int block_size,
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
    key_cache[dst] = quantize16(key[2 * i], key[2 * i + 1], __ldg(k_scale + h));
    value_cache[dst] = quantize16(value[2 * i], value[2 * i + 1], __ldg(v_scale + h));
  }
}

// swap_blocks: grid-stride over (pair, 16-byte chunk); each thread keeps 4 loads in
// flight before its stores, so reads across the host link overlap.
__global__ void __launch_bounds__(256) swap_blocks_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                          const int64_t* __restrict__ block_mapping, int num_pairs,
                                                          int src_blocks, int dst_blocks, int64_t chunks_per_block,
                                                          int32_t* status) {
  const int64_t total = static_cast<int64_t>(num_pairs) * chunks_per_block;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  constexpr int kUnroll = 4;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; base < total;
       base += stride * kUnroll) {
    uint4 v[kUnroll];
    int64_t to[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      to[u] = -1;
      const int64_t i = base + u * stride;
      if (i >= total) continue;
      const int64_t pair = i / chunks_per_block, c = i - pair * chunks_per_block;
      const int64_t s = block_mapping[2 * pair], d = block_mapping[2 * pair + 1];
      if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks) {
        if (c == 0) set_status(status, PKV_DEV_BAD_PAIR);
        continue;
      }
      v[u] = src[s * chunks_per_block + c];
      to[u] = d * chunks_per_block + c;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (to[u] >= 0) dst[to[u]] = v[u];
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

extern "C" int pkv_reshape_and_cache_fp8(const void* key, const void* value, void* key_cache, void* value_cache,
                                         const int64_t* slot_mapping, const float* k_scale, const float* v_scale,
                                         int num_tokens, int num_blocks, int num_kv_heads, int head_dim,
                                         int block_size, int32_t* status, pkv_stream_t stream) {
  clear_error();
  if (num_tokens < 0 || num_blocks <= 0 || num_kv_heads <= 0)
    return set_error(PKV_ERR_INVALID, "reshape_and_cache_fp8: bad sizes");
  if (head_dim != 64 && head_dim != 128)
    return set_error(PKV_ERR_UNSUPPORTED, "reshape_and_cache_fp8: head_dim %d not in {64,128}", head_dim);
  if (block_size != 16 && block_size != 32)
    return set_error(PKV_ERR_UNSUPPORTED, "reshape_and_cache_fp8: block_size %d not in {16,32}", block_size);
  if (num_tokens == 0) return PKV_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping || !k_scale || !v_scale)
    return set_error(PKV_ERR_INVALID, "reshape_and_cache_fp8: null pointer");
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
    return set_error(PKV_ERR_INVALID, "reshape_and_cache_fp8: tensors must be 16-byte aligned");
  const int chunks_per_row = head_dim / 16;
  const int64_t total = static_cast<int64_t>(num_tokens) * num_kv_heads * chunks_per_row;
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int blocks = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(sm_count()) * 8));
  reshape_and_cache_fp8_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(key), static_cast<const uint4*>(value), static_cast<uint4*>(key_cache),
      static_cast<uint4*>(value_cache), slot_mapping, k_scale, v_scale, total, chunks_per_row, num_kv_heads,
      block_size, static_cast<int64_t>(num_blocks) * block_size, status);
  return check_launch("reshape_and_cache_fp8 launch");
}

extern "C" int pkv_swap_blocks(const void* src_pool, void* dst_pool, const int64_t* block_mapping, int num_pairs,
                               int src_blocks, int dst_blocks, int64_t block_bytes, int32_t* status,
                               pkv_stream_t stream) {
  clear_error();
  if (num_pairs < 0 || src_blocks <= 0 || dst_blocks <= 0 || block_bytes <= 0)
    return set_error(PKV_ERR_INVALID, "swap_blocks: bad sizes");
  if (block_bytes % 16 != 0) return set_error(PKV_ERR_INVALID, "swap_blocks: block bytes must be a multiple of 16");
  if (num_pairs == 0) return PKV_OK;
  if (!src_pool || !dst_pool || !block_mapping) return set_error(PKV_ERR_INVALID, "swap_blocks: null pointer");
  if (!aligned16(src_pool) || !aligned16(dst_pool))
    return set_error(PKV_ERR_INVALID, "swap_blocks: pools must be 16-byte aligned");
  // Every pointer the kernel dereferences must be device memory or pinned host
  // memory mapped into the device's address space.
  const void* ptrs[3] = {src_pool, dst_pool, block_mapping};
  const char* names[3] = {"src_pool", "dst_pool", "block_mapping"};
  for (int i = 0; i < 3; ++i) {
    cudaPointerAttributes attr{};
    if (cudaPointerGetAttributes(&attr, ptrs[i]) != cudaSuccess) {
      cudaGetLastError();
      return set_error(PKV_ERR_INVALID, "swap_blocks: %s is not CUDA-visible memory", names[i]);
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeHost && attr.type != cudaMemoryTypeManaged)
      return set_error(PKV_ERR_INVALID, "swap_blocks: %s must be device or pinned host memory", names[i]);
    if (attr.type == cudaMemoryTypeHost && attr.devicePointer != ptrs[i])
      return set_error(PKV_ERR_INVALID, "swap_blocks: pinned %s is not mapped at the same address on the device",
                       names[i]);
  }
  const int64_t chunks = block_bytes / 16;
  const int64_t total = chunks * num_pairs;
  const int threads = 256;
  const int64_t want = (total + threads * 4 - 1) / (threads * 4);
  const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, static_cast<int64_t>(sm_count()) * 8)));
  swap_blocks_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src_pool), static_cast<uint4*>(dst_pool), block_mapping, num_pairs, src_blocks,
      dst_blocks, chunks, status);
  return check_launch("swap_blocks launch");
}
