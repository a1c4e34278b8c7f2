// Decode attention for callers that cannot allocate device memory.
//
// pkv_paged_attention_decode needs a caller-provided device workspace (the work
// plan, the split-partition partials and their arrival counters).  Some callers
// have no way to provide one: a host runtime's custom-operator interface may hand
// a plugin its input and output tensors and nothing else, and some applications
// reserve all device memory up front for their own allocator or forbid device
// allocations once they are running.  This file gives them a variant whose scratch
// lives in a fixed array compiled into the library.
//
// The array is a file-scope __device__ variable, so every GPU on which the library
// is loaded holds PKV_STATIC_SCRATCH_BYTES of it until the process exits.  Host
// code must not pass the array's name to a kernel (on the host that name is only a
// stand-in, not a device address): the device address is looked up once per device
// with cudaGetSymbolAddress, with that device current, on the first call made
// there.  That first call on each device should therefore happen before any stream
// capture begins.  With CUDA's lazy module loading (the default) the array itself is
// also placed in device memory only then, so an application that hands all device
// memory to its own allocator should make the first call before it does.  The
// looked-up address is kept for the life of the process: after a device reset
// (cudaDeviceReset) it is stale, so this entry point must not be used on that device
// again.  All calls on a device share the one array and it keeps the
// previous call's contents; the plan kernel re-zeroes everything that must start
// at zero on every call, but two calls whose kernels overlap on the GPU (for
// example on two streams) race on the array and corrupt each other's results.
#include <cuda_runtime.h>

#include <mutex>

#include "decode_common.cuh"
#include "pkv_internal.h"

namespace pkv {

static __device__ __align__(256) unsigned char g_static_scratch[PKV_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
static std::mutex g_static_mutex;
static void* g_static_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
static int static_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "decode_static: cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return set_error(PKV_ERR_INVALID, "decode_static: device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p)
      return set_error(PKV_ERR_CUDA, "decode_static: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return PKV_OK;
}

}  // namespace pkv

extern "C" int pkv_paged_attention_decode_static(void* out, int out_dtype, const void* query, const void* key_cache,
                                                 const void* value_cache, const int32_t* block_tables,
                                                 int max_blocks_per_seq, const int32_t* context_lens,
                                                 int max_context_len, int num_seqs, int num_heads, int num_kv_heads,
                                                 int head_dim, int block_size, int num_blocks, float scale,
                                                 int partition_tokens, int path, int32_t* status,
                                                 pkv_stream_t stream) {
  using namespace pkv;
  clear_error();
  // Sizes the workspace variant refuses give its return code, before the scratch is looked up.
  int partition = 0;
  const int rc_sizes = decode_check_sizes(out_dtype, false, max_blocks_per_seq, max_context_len, num_seqs, num_heads,
                                          num_kv_heads, head_dim, block_size, num_blocks, partition_tokens, path,
                                          &partition);
  if (rc_sizes != PKV_OK) return rc_sizes;
  if (num_seqs == 0) return PKV_OK;
  const size_t need = pkv_paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                         max_context_len, partition_tokens);
  if (need == 0) return set_error(PKV_ERR_INVALID, "paged_attention_decode_static: bad sizes");
  if (need > static_cast<size_t>(PKV_STATIC_SCRATCH_BYTES))
    return set_error(PKV_ERR_INVALID,
                     "paged_attention_decode_static: these sizes need %zu bytes of scratch, more than the %zu-byte "
                     "built-in array; use pkv_paged_attention_decode with a workspace",
                     need, static_cast<size_t>(PKV_STATIC_SCRATCH_BYTES));
  void* scratch = nullptr;
  int rc = static_scratch_address(&scratch);
  if (rc != PKV_OK) return rc;
  return pkv_paged_attention_decode(out, out_dtype, query, key_cache, value_cache, block_tables, max_blocks_per_seq,
                                    context_lens, max_context_len, num_seqs, num_heads, num_kv_heads, head_dim,
                                    block_size, num_blocks, scale, partition_tokens, path, scratch,
                                    static_cast<size_t>(PKV_STATIC_SCRATCH_BYTES), status, stream);
}
