// Shared definitions of the decode-attention kernels: launch arguments, the
// work plan (entries of (sequence, partition) sorted longest first) and the
// workspace layout.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "device_common.cuh"

namespace pkv {

// Tokens that one pipeline stage carries: one 16-row slice of a (block, kv head)
// tile (a whole block at block_size 16, half a block at 32).
constexpr int kStageTokens = 16;
constexpr int kMaxPartition = 2048;       // the tensor-core path reads up to 128 table entries per item
constexpr int kMaxPartitionSimt = 512;    // the CUDA-core path keeps one table entry per lane (32 blocks)
constexpr int kPlanBuckets = 513;         // counting-sort buckets of the plan (item length, coarsened)

// One plan entry: a (sequence, partition) pair.  x = seq, y = partition index,
// z = number of partitions of the sequence, w = validated context length.
using PlanEntry = int4;

struct DecodeArgs {
  void* out;
  const __nv_bfloat16* query;
  const __nv_bfloat16* key_cache;
  const __nv_bfloat16* value_cache;
  const uint8_t* key_cache8;   // 8-bit (e4m3) pools of the fp8 entry point, else null
  const uint8_t* value_cache8;
  const float* k_scale;        // [num_kv_heads] scales of the 8-bit pools
  const float* v_scale;
  const int32_t* block_tables;
  const int32_t* plan_count;   // [0] number of plan entries, [1] work-item counter (both set by the plan kernel)
  const PlanEntry* entries;    // sorted plan
  int32_t* arrive;             // [B * Hq] partition arrival counters (zeroed by the plan kernel)
  float* part_o;               // [B * Hq * max_parts * D] unnormalised partial outputs
  float2* part_ml;             // [B * Hq * max_parts] (running max in log2 units, sum of weights)
  int32_t* status;
  const int32_t* context_lens;
  int max_context_len;
  int max_blocks;
  int num_seqs;
  int num_heads;
  int num_kv_heads;
  int block_size;
  int num_blocks;
  int group;                   // num_heads / num_kv_heads
  int partition;               // tokens per partition
  int max_parts;
  float scale_log2;            // scale * log2(e): scores are kept in base-2 units
  // Shared-prefix decode, private phase (tensor-core path only): each row's table is read from
  // position block_offset[row] on, and every item writes its partial (o, m, l), also unsplit
  // ones; the merge of the shared-prefix decode combines them.  Null / 0 otherwise.
  const int32_t* block_offset;
  int always_partial;
  // 8-bit tensor-core path: the queries split once per call into e4m3 [hi; lo] rows (32 rows of
  // 128 codes per (sequence, kv head)) and the power of two 2^-e of each head (16 per unit).
  uint8_t* q_split;
  float* q_inv;
};

// Workspace layout, identical for every decode path.
struct WorkspaceLayout {
  int partition = 0;
  int max_parts = 0;
  size_t off_count = 0, off_arrive = 0, off_entries = 0, off_part_o = 0, off_part_ml = 0, total = 0;
  size_t off_qsplit = 0, off_qinv = 0;  // only when the tensor-core path can run (split queries of the 8-bit pool)
};

// Bytes of split queries per (sequence, kv head) unit: 32 rows of 128 e4m3 codes, and 16 scales.
constexpr size_t kQSplitUnitBytes = 32 * 128;
constexpr size_t kQInvUnitBytes = 16 * sizeof(float);
bool tensor_path_supports(int group, int head_dim);

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

#ifndef PKV_SIMT_MIN_ITEMS
#define PKV_SIMT_MIN_ITEMS 16384
#endif
inline int auto_partition_tokens(int num_seqs, int num_kv_heads, int block_size, int max_context_len) {
  // Largest split (fewest partials to merge) that still leaves enough work items to keep
  // every warp of the GPU busy to the end (148 SMs x 12 warps; items are taken longest
  // first).  The 7B batch (64 x U{10..2000}, 32 heads) gets 256-token splits, ~9,000
  // items: 6,020 -> 6,336 GB/s against 512-token splits; batches with more (sequence,
  // head) units keep 512.
  int p = kMaxPartitionSimt;
  while (p > 64 && static_cast<int64_t>(num_seqs) * num_kv_heads * ((max_context_len + p - 1) / p) < PKV_SIMT_MIN_ITEMS)
    p /= 2;
  return p < block_size ? block_size : p;
}

// The tensor-core path pays a fixed cost per item (the first tile's maximum, the
// output or partial, and later a merge): it takes longer splits, up to 2048 tokens, as
// long as about 8 items per SM remain for load balance (long-context batch, 16 x
// U{5k..32k}: 2048-token splits, 5,764 -> 5,852 GB/s bf16 and 5,107 -> 5,348 e4m3
// against the 1024 that a target of 16 per SM gave; 32 per SM was slower still).  With at least 4 (sequence,
// kv head) units per SM it never splits below 512 tokens: items of one or two tiles
// would cost about as much in per-item work as in streaming, and the units alone
// balance the SMs.  Never shorter than the CUDA-core split, so a workspace sized for
// that split always suffices.
#ifndef PKV_TC_ITEMS_PER_SM
#define PKV_TC_ITEMS_PER_SM 8
#endif
inline int auto_partition_tokens_tensor(int num_seqs, int num_kv_heads, int block_size, int max_context_len) {
  const int base = auto_partition_tokens(num_seqs, num_kv_heads, block_size, max_context_len);
  const int64_t units = static_cast<int64_t>(num_seqs) * num_kv_heads;
  int p = kMaxPartition;
  while (p > base && units * ((max_context_len + p - 1) / p) < PKV_TC_ITEMS_PER_SM * 148) p /= 2;
  if (units >= 4 * 148 && p < 512) p = 512;
  return p > base ? p : base;
}

inline WorkspaceLayout workspace_layout(int num_seqs, int num_heads, int head_dim, int max_context_len,
                                        int partition, bool force_partials = false, int num_kv_heads = 0) {
  WorkspaceLayout w;
  w.partition = partition;
  w.max_parts = max_context_len <= 0 ? 1 : (max_context_len + partition - 1) / partition;
  size_t off = 0;
  w.off_count = off;
  off = align256(off + sizeof(int32_t));
  w.off_arrive = off;
  off = align256(off + static_cast<size_t>(num_seqs) * num_heads * sizeof(int32_t));
  w.off_entries = off;
  off = align256(off + static_cast<size_t>(num_seqs) * w.max_parts * sizeof(PlanEntry));
  w.off_part_o = off;
  if (w.max_parts > 1 || force_partials) {
    off = align256(off + static_cast<size_t>(num_seqs) * num_heads * w.max_parts * head_dim * sizeof(float));
    w.off_part_ml = off;
    off = align256(off + static_cast<size_t>(num_seqs) * num_heads * w.max_parts * sizeof(float2));
  } else {
    w.off_part_ml = off;
  }
  if (num_kv_heads > 0 && num_heads % num_kv_heads == 0 && tensor_path_supports(num_heads / num_kv_heads, head_dim)) {
    const size_t units = static_cast<size_t>(num_seqs) * num_kv_heads;
    w.off_qsplit = off;
    off = align256(off + units * kQSplitUnitBytes);
    w.off_qinv = off;
    off = align256(off + units * kQInvUnitBytes);
  }
  w.total = off;
  return w;
}

// The shared phase of the shared-prefix decode: the prefill kernel in segment mode over the
// plan's entries and parts (prefill_tc.cu).
struct SegmentLaunch {
  const void* query;            // [num_seqs, num_heads, 128] bf16
  const void* key_cache;
  const void* value_cache;
  const int32_t* block_tables;
  const int32_t* plan_count;    // [0] entries, [1] work-item counter (zero before the launch)
  const int4* entries;
  const int4* parts;
  float* part_o;
  float2* part_ml;
  int32_t* status;
  int num_entries;              // grid sizing (host)
  int max_blocks, num_seqs, num_heads, num_kv_heads, block_size, num_blocks;
  float scale;
  // pools of widened 8-bit codes: per-kv-head factors of the scores and of the partial
  // outputs (null for bf16 pools)
  const float* k_scale = nullptr;
  const float* v_scale = nullptr;
};
int launch_prefill_segments(const SegmentLaunch& launch, cudaStream_t stream);

// Launchers living in other translation units.
// The decode plan kernel (decode.cu): validates context_lens, sorts (sequence, partition)
// entries longest first into a.entries, zeroes a.plan_count's counter and a.arrive.
int launch_decode_plan(const DecodeArgs& a, const int32_t* context_lens, int max_context_len, cudaStream_t stream);
int launch_decode_tensor(const DecodeArgs& a, int head_dim, bool out_f32, cudaStream_t stream);
// The CUDA-core decode (bf16 pools, or 8-bit ones when a.key_cache8 is set; decode.cu).
int launch_decode_simt(const DecodeArgs& a, int head_dim, bool out_f32, cudaStream_t stream);
int launch_decode_tensor_fp8(const DecodeArgs& a, int head_dim, bool out_f32, cudaStream_t stream);
// Merge of split partitions (no launch when max_parts <= 1), after a tensor-core decode.
int launch_merge_partials(const DecodeArgs& a, bool out_f32, cudaStream_t stream);

}  // namespace pkv
