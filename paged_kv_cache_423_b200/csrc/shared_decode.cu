// Shared-prefix decode: the run of a plan made by pkv_shared_plan (shared_plan.cpp).
//
// Blocks that adjacent rows hold in common (a shared system prompt, a parent's blocks in
// its beams; Outcome School explainer, "内存共享") are attended to once per kv head for
// all of those rows, as one dense contraction on the tensor cores; each row's private
// remainder goes through the tensor-core decode; a merge combines the partial results
// by log-sum-exp rescaling, which reproduces softmax attention over the whole context
// (intelliparadigm article "PagedAttention：操作系统分页思想的跨界创新" §2.1).
//
// Launches, on the caller's stream unless noted:
//   shared_setup_kernel   checks the plan against the call (sizes, ranges, that every
//                         row's shared tokens plus its remainder equal its context
//                         length) and writes checked copies of the remainders; a plan
//                         that does not fit sets PKV_DEV_BAD_CONTEXT and every output
//                         row becomes zero
//   prefill_tc_kernel     segment mode, on a side stream forked after the set-up: all query
//                         heads of a part's rows against the part's keys, unnormalised
//                         partials (o, m, l)
//   plan_kernel +
//   decode_gqa_tc_kernel  the remainders, every item writing its partial, beside the shared
//                         phase (the two write disjoint partials, and each kernel's CTAs take
//                         the SMs the other leaves)
//   shared_merge_kernel   after both (the side stream joins back): out = sum 2^(m_i - M) o_i /
//                         sum 2^(m_i - M) l_i per (row, head)
// Over an 8-bit (e4m3) pool the shared phase first widens the codes of every part's blocks
// into bf16 scratch pools (scratch_fill_kernel, on the side stream: exact, every e4m3 value
// is a bf16 value) and runs on them with the kv head's key scale folded into its score scale
// and its value scale into its partial outputs; the private phase is the 8-bit tensor-core
// decode.
// The side stream and its two events are created on the first call on each device and kept
// until the process exits; the enqueue of a call is serialised per device, so calls from
// several host threads stay correct.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "decode_common.cuh"
#include "per_device.h"
#include "pkv_internal.h"

namespace pkv {
namespace sp {

constexpr int kD = 128;
constexpr int kSetupThreads = 1024;
// Private remainders of at most this many tokens (one tile of the tensor-core decode) go
// through the CUDA-core decode (a warp per (row, query head, partition), little fixed work per
// item), longer ones through the tensor-core decode (one item per (row, kv head, partition),
// tiles of 128 tokens).  Measured on the shared-prompt batch forked into 4 beams (remainders of
// at most 32 tokens) the CUDA-core phase is faster; with the prompt batch's remainders of up to
// 500 tokens the tensor-core one is.
#ifndef PKV_SHARED_SIMT_MAX
#define PKV_SHARED_SIMT_MAX 128
#endif
constexpr int kSimtSuffixMax = PKV_SHARED_SIMT_MAX;
constexpr int kMergeWarps = 4;

struct Layout {
  size_t off_count = 0, off_lens = 0, off_offset = 0, off_seg_o = 0, off_seg_ml = 0, off_decode = 0, total = 0;
  size_t off_scr_k = 0, off_scr_v = 0, off_scr_tab = 0;  // 8-bit pools only
  int64_t scratch_blocks = 0;
  WorkspaceLayout dec;
  int partition = 0;
  bool private_simt = false;  // the private phase on the CUDA-core decode
};

// Workspace: [plan count, work counter, bad flag] | checked remainders | checked block offsets |
// shared partials (o, then (m, l)) | the private phase's decode workspace (partials forced) |
// 8-bit pools: the widened K and V scratch pools [scratch block][kv head][block_size][128] bf16
// and their table [num_seqs][max_blocks] (written where a part's blocks sit in the call's table).
static Layout layout(const pkv_shared_plan_info& in, int num_heads, int num_kv_heads, bool kv8) {
  Layout L;
  const int B = in.num_seqs;
  L.private_simt = in.max_suffix_len <= kSimtSuffixMax;
  L.partition = L.private_simt ? auto_partition_tokens(B, num_kv_heads, in.block_size, in.max_suffix_len)
                               : auto_partition_tokens_tensor(B, num_kv_heads, in.block_size, in.max_suffix_len);
  size_t off = 0;
  L.off_count = off;
  off = align256(off + 4 * sizeof(int32_t));
  L.off_lens = off;
  off = align256(off + static_cast<size_t>(B) * sizeof(int32_t));
  L.off_offset = off;
  off = align256(off + static_cast<size_t>(B) * sizeof(int32_t));
  L.off_seg_o = off;
  off = align256(off + static_cast<size_t>(in.num_partials) * num_heads * kD * sizeof(float));
  L.off_seg_ml = off;
  off = align256(off + static_cast<size_t>(in.num_partials) * num_heads * sizeof(float2));
  L.off_decode = off;
  L.dec = workspace_layout(B, num_heads, kD, in.max_suffix_len, L.partition, true, kv8 ? num_kv_heads : 0);
  off = align256(off + L.dec.total);
  if (kv8) {
    L.scratch_blocks = in.block_size > 0 ? in.shared_tokens / in.block_size : 0;
    const size_t pool = static_cast<size_t>(L.scratch_blocks) * num_kv_heads * in.block_size * kD * 2;
    L.off_scr_k = off;
    off = align256(off + pool);
    L.off_scr_v = off;
    off = align256(off + pool);
    L.off_scr_tab = off;
    off = align256(off + static_cast<size_t>(B) * in.max_blocks_per_seq * sizeof(int32_t));
  }
  L.total = off;
  return L;
}

struct SetupArgs {
  const int4* entries;
  const int4* parts;
  const int32_t* suffix_lens;
  const int32_t* block_offset;
  const int32_t* row_start;
  const int32_t* row_ids;
  const int32_t* context_lens;
  int32_t* count;          // [0] shared-phase entries, [1] its work counter, [2] bad plan
  int32_t* v_lens;         // checked remainders (0 for every row of a bad plan)
  int32_t* v_offset;
  int32_t* status;
  int num_seqs, num_entries, num_parts, num_partials, max_blocks, block_size, tile_rows, max_suffix_len;
  int64_t scratch_blocks;  // 8-bit run: the scratch pools' blocks (each part's base is checked), else -1
};

__global__ void __launch_bounds__(kSetupThreads) shared_setup_kernel(const SetupArgs p) {
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  bool mine = false;
  for (int i = threadIdx.x; i < p.num_parts; i += blockDim.x) {
    const int4 d0 = p.parts[2 * i], d1 = p.parts[2 * i + 1];
    const int64_t nblk = d0.z >= 1 ? (static_cast<int64_t>(d0.z) + p.block_size - 1) / p.block_size : 0;
    mine |= d0.x < 0 || d0.x >= p.num_seqs || d0.y < 0 || d0.z < 1 || d0.y + nblk > p.max_blocks || d0.w < 0 ||
            d1.x < 1 || static_cast<int64_t>(d0.w) + d1.x > p.num_seqs || d1.y < 0 ||
            static_cast<int64_t>(d1.y) + d1.x > p.num_partials;
    if (p.scratch_blocks >= 0) mine |= d0.z % p.block_size != 0 || d1.z < 0 || d1.z + nblk > p.scratch_blocks;
  }
  for (int i = threadIdx.x; i < p.num_entries; i += blockDim.x) {
    const int4 e = p.entries[i];
    if (e.w < 0 || e.w >= p.num_parts) {
      mine = true;
      continue;
    }
    const int4 d0 = p.parts[2 * e.w], d1 = p.parts[2 * e.w + 1];
    const int na = e.z & 0xff, nb = (e.z >> 8) & 0xff;
    mine |= (e.z >> 16) != 0 || na < 1 || na > p.tile_rows || nb > p.tile_rows || (nb > 0 && na != p.tile_rows) ||
            e.x < d0.w || static_cast<int64_t>(e.x) + na + nb > static_cast<int64_t>(d0.w) + d1.x;
  }
  for (int r = threadIdx.x; r < p.num_seqs; r += blockDim.x) {
    const int off = p.block_offset[r], sl = p.suffix_lens[r], L = p.context_lens[r];
    const bool ok = off >= 0 && off <= p.max_blocks && sl >= 0 && sl <= p.max_suffix_len &&
                    static_cast<int64_t>(sl) <= static_cast<int64_t>(p.max_blocks - off) * p.block_size &&
                    static_cast<int64_t>(off) * p.block_size + sl == L;
    mine |= !ok;
    const int a = p.row_start[r], b = p.row_start[r + 1];
    mine |= a < 0 || b < a || b > p.num_partials || (r == 0 && a != 0) ||
            (r == p.num_seqs - 1 && b != p.num_partials);
    if (a >= 0 && b <= p.num_partials)
      for (int k = a; k < b; ++k) mine |= p.row_ids[k] < 0 || p.row_ids[k] >= p.num_partials;
  }
  if (mine) atomicOr(&bad, 1);
  __syncthreads();
  for (int r = threadIdx.x; r < p.num_seqs; r += blockDim.x) {
    p.v_lens[r] = bad ? 0 : p.suffix_lens[r];
    p.v_offset[r] = bad ? 0 : p.block_offset[r];
  }
  if (threadIdx.x == 0) {
    p.count[0] = bad ? 0 : p.num_entries;
    p.count[1] = 0;
    p.count[2] = bad;
    if (bad) set_status(p.status, PKV_DEV_BAD_CONTEXT);
  }
}

// ---- 8-bit pools: the shared phase's blocks widened into bf16 scratch pools
struct ScratchArgs {
  const int4* parts;
  const int32_t* block_tables;
  const uint8_t* key8;
  const uint8_t* value8;
  __nv_bfloat16* key_s;
  __nv_bfloat16* value_s;
  int32_t* table_s;
  const int32_t* bad;   // the set-up's verdict on the plan
  int32_t* status;
  int num_parts, num_seqs, max_blocks, block_size, num_blocks, num_kv_heads;
  int64_t scratch_blocks;
};

constexpr int kScratchThreads = 256;
constexpr int kScratchSplit = 4;  // CTAs sharing one (part, kv head)

// Four e4m3 codes (low byte first) as four bf16 values, exactly (through f16, which holds
// every e4m3 value; so does bf16).
__device__ __forceinline__ uint2 e4m3x4_to_bf16x4(uint32_t w) {
  uint32_t h01, h23;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(h01), "=r"(h23)
      : "r"(w));
  const __half2 a = *reinterpret_cast<const __half2*>(&h01), b = *reinterpret_cast<const __half2*>(&h23);
  return make_uint2(pack_bf16x2(__low2float(a), __high2float(a)), pack_bf16x2(__low2float(b), __high2float(b)));
}

// CTA (part, kv head, z) widens blocks z, z + kScratchSplit, .. of the part for one kv head
// into scratch blocks base + j, and (kv head 0) points the scratch table's entry of the block
// at it, or at -1 for a table entry outside the pool (the shared phase then flags
// PKV_DEV_BAD_BLOCK and masks its keys, as over a bf16 pool).
__global__ void __launch_bounds__(kScratchThreads) scratch_fill_kernel(const ScratchArgs p) {
  if (*p.bad) return;
  const int part = blockIdx.x, kvh = blockIdx.y;
  const int4 d0 = p.parts[2 * part], d1 = p.parts[2 * part + 1];
  const int row = d0.x, pos0 = d0.y, nblk = d0.z / p.block_size, base = d1.z;
  if (row < 0 || row >= p.num_seqs || pos0 < 0 || nblk < 0 || pos0 + nblk > p.max_blocks || base < 0 ||
      base + static_cast<int64_t>(nblk) > p.scratch_blocks) {
    if (threadIdx.x == 0 && kvh == 0 && blockIdx.z == 0) set_status(p.status, PKV_DEV_BAD_CONTEXT);
    return;
  }
  const int codes = p.block_size * kD;  // one (block, kv head) tile
  for (int j = blockIdx.z; j < nblk; j += gridDim.z) {
    const int64_t tpos = static_cast<int64_t>(row) * p.max_blocks + pos0 + j;
    const int phys = p.block_tables[tpos];
    const bool ok = phys >= 0 && phys < p.num_blocks;
    if (kvh == 0 && threadIdx.x == 0) p.table_s[tpos] = ok ? base + j : -1;
    if (!ok) continue;
    const int64_t src = (static_cast<int64_t>(phys) * p.num_kv_heads + kvh) * codes;
    const int64_t dst = (static_cast<int64_t>(base + j) * p.num_kv_heads + kvh) * codes;
    const uint4* ks = reinterpret_cast<const uint4*>(p.key8 + src);
    const uint4* vs = reinterpret_cast<const uint4*>(p.value8 + src);
    uint4* kd = reinterpret_cast<uint4*>(p.key_s + dst);
    uint4* vd = reinterpret_cast<uint4*>(p.value_s + dst);
    for (int i = threadIdx.x; i < codes / 16; i += blockDim.x) {  // 16 codes -> 32 bytes
      const uint4 kw = __ldg(ks + i), vw = __ldg(vs + i);
      uint2 a = e4m3x4_to_bf16x4(kw.x), b = e4m3x4_to_bf16x4(kw.y), c = e4m3x4_to_bf16x4(kw.z),
            d = e4m3x4_to_bf16x4(kw.w);
      kd[2 * i] = make_uint4(a.x, a.y, b.x, b.y);
      kd[2 * i + 1] = make_uint4(c.x, c.y, d.x, d.y);
      a = e4m3x4_to_bf16x4(vw.x), b = e4m3x4_to_bf16x4(vw.y), c = e4m3x4_to_bf16x4(vw.z), d = e4m3x4_to_bf16x4(vw.w);
      vd[2 * i] = make_uint4(a.x, a.y, b.x, b.y);
      vd[2 * i + 1] = make_uint4(c.x, c.y, d.x, d.y);
    }
  }
}

// The side stream of the shared phase and the fork / join events, one set per device.
struct Side {
  cudaStream_t stream;
  cudaEvent_t fork, join;
};
static PerDevice<Side> g_side;
static std::mutex g_side_mutex[kMaxDevices];

static int side_for(int dev, Side* out) {
  return g_side.get(
      dev,
      [](Side& s) {
        cudaError_t e = cudaStreamCreateWithFlags(&s.stream, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming);
        return static_cast<int>(e);
      },
      out, static_cast<int>(cudaErrorInvalidDevice));
}

struct MergeArgs {
  void* out;
  const float* dec_o;       // private phase partials [row * Hq + h][max_parts][128]
  const float2* dec_ml;
  const float* seg_o;       // shared partials [id][h][128]
  const float2* seg_ml;
  const int32_t* v_lens;
  const int32_t* row_start;
  const int32_t* row_ids;
  const int32_t* bad;
  int num_seqs, num_heads, partition, max_parts;
};

// One warp per (row, head); lane l owns output values 4l .. 4l+3.
template <bool OUT_F32>
__global__ void __launch_bounds__(kMergeWarps * 32) shared_merge_kernel(const MergeArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t unit = static_cast<int64_t>(blockIdx.x) * kMergeWarps + warp;
  if (unit >= static_cast<int64_t>(a.num_seqs) * a.num_heads) return;
  const int r = static_cast<int>(unit / a.num_heads), h = static_cast<int>(unit % a.num_heads);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float Ls = 0.f;
  if (*a.bad == 0) {
    const int sl = a.v_lens[r];
    const int np = sl == 0 ? 1 : (sl + a.partition - 1) / a.partition;
    const int s0 = a.row_start[r], s1 = a.row_start[r + 1];
    const float2* dml = a.dec_ml + unit * a.max_parts;
    float M = -INFINITY;
    for (int p = lane; p < np; p += 32) M = fmaxf(M, dml[p].x);
    for (int k = s0 + lane; k < s1; k += 32) M = fmaxf(M, a.seg_ml[static_cast<int64_t>(a.row_ids[k]) * a.num_heads + h].x);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    auto add = [&](float2 ml, const float* o) {
      const float w = ml.x == -INFINITY ? 0.f : exp2f(ml.x - M);
      Ls = fmaf(w, ml.y, Ls);
      const float4 v = *reinterpret_cast<const float4*>(o + lane * 4);
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    };
    for (int p = 0; p < np; ++p) add(dml[p], a.dec_o + (unit * a.max_parts + p) * kD);
    for (int k = s0; k < s1; ++k) {
      const int64_t id = static_cast<int64_t>(a.row_ids[k]) * a.num_heads + h;
      add(a.seg_ml[id], a.seg_o + id * kD);
    }
  }
  const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
  const int64_t o = unit * kD + lane * 4;
  if constexpr (OUT_F32) {
    *reinterpret_cast<float4*>(static_cast<float*>(a.out) + o) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  } else {
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + o) =
        make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
  }
}

}  // namespace sp
}  // namespace pkv

using namespace pkv;

static size_t shared_workspace_size(const pkv_shared_plan_info* info, int num_heads, int num_kv_heads, int head_dim,
                                    bool kv8) {
  if (!info || info->num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim != sp::kD ||
      info->num_partials < 0 || info->max_suffix_len < 0 || (info->block_size != 16 && info->block_size != 32) ||
      info->shared_tokens < 0 || info->max_blocks_per_seq <= 0)
    return 0;
  return sp::layout(*info, num_heads, num_kv_heads, kv8).total;
}

extern "C" size_t pkv_paged_attention_decode_shared_workspace_size(const pkv_shared_plan_info* info, int num_heads,
                                                                   int num_kv_heads, int head_dim) {
  return shared_workspace_size(info, num_heads, num_kv_heads, head_dim, false);
}

extern "C" size_t pkv_paged_attention_decode_shared_fp8_workspace_size(const pkv_shared_plan_info* info,
                                                                       int num_heads, int num_kv_heads,
                                                                       int head_dim) {
  return shared_workspace_size(info, num_heads, num_kv_heads, head_dim, true);
}

// kv8: the pools hold e4m3 codes with per-kv-head scales k_scale / v_scale.
static int shared_impl(bool kv8, void* out, int out_dtype, const void* query, const void* key_cache,
                       const void* value_cache, const float* k_scale, const float* v_scale,
                       const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                       int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                       const void* plan, const pkv_shared_plan_info* info, void* workspace, size_t workspace_bytes,
                       int32_t* status, pkv_stream_t stream) {
  if (!info) return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: null info");
  const pkv_shared_plan_info& in = *info;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0)
    return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: bad sizes");
  if (out_dtype != PKV_DTYPE_BF16 && out_dtype != PKV_DTYPE_F32)
    return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: out_dtype %d", out_dtype);
  if (block_size != 16 && block_size != 32)
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_decode_shared: block_size %d not in {16,32}", block_size);
  if (num_heads % num_kv_heads != 0 || !tensor_path_supports(num_heads / num_kv_heads, head_dim))
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_decode_shared: needs head_dim 128 and 2 <= num_heads / "
                     "num_kv_heads <= 16 (got %d, %d / %d)", head_dim, num_heads, num_kv_heads);
  if (num_kv_heads >= (1 << 15))
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_decode_shared: num_kv_heads %d", num_kv_heads);
  if (!(scale > 0.f) || !std::isfinite(scale))  // the shared phase masks keys with -inf scores
    return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: scale must be finite and positive");
  const int group = num_heads / num_kv_heads;
  if (in.num_seqs != num_seqs || in.group != group || in.block_size != block_size ||
      in.max_blocks_per_seq != max_blocks_per_seq || in.num_entries < 0 || in.num_parts < 0 ||
      in.num_partials < 0 || in.max_suffix_len < 0 || in.max_suffix_len > max_blocks_per_seq * block_size)
    return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: the plan was made for other sizes");
  if (static_cast<int64_t>(num_blocks) * num_kv_heads * block_size > (static_cast<int64_t>(1) << 31))
    return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: pool too large");
  if (static_cast<int64_t>(in.num_entries) * num_kv_heads > (int64_t{1} << 30))
    return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: too many shared-phase entries");
  if (num_seqs == 0) return PKV_OK;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens || !plan || !workspace ||
      (kv8 && (!k_scale || !v_scale)))
    return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: null pointer");
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) || !aligned16(plan))
    return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: tensors and the plan must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: workspace must be 256-byte aligned");
  const uint64_t offs[] = {in.off_entries, in.off_parts, in.off_suffix_lens, in.off_block_offset, in.off_row_start,
                           in.off_row_ids};
  for (uint64_t o : offs)
    if (o % 16 != 0 || o > in.bytes) return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: bad plan offsets");
  if (in.off_entries + static_cast<uint64_t>(in.num_entries) * 16 > in.bytes ||
      in.off_parts + static_cast<uint64_t>(in.num_parts) * 32 > in.bytes ||
      in.off_suffix_lens + static_cast<uint64_t>(num_seqs) * 4 > in.bytes ||
      in.off_block_offset + static_cast<uint64_t>(num_seqs) * 4 > in.bytes ||
      in.off_row_start + static_cast<uint64_t>(num_seqs + 1) * 4 > in.bytes ||
      in.off_row_ids + static_cast<uint64_t>(in.num_partials) * 4 > in.bytes)
    return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: plan sections exceed its size");
  if (in.shared_tokens < 0 || in.shared_tokens % block_size != 0 ||
      (kv8 && in.shared_tokens / block_size * num_kv_heads * block_size > (int64_t{1} << 31)))
    return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: bad shared token count in the plan info");
  const sp::Layout L = sp::layout(in, num_heads, num_kv_heads, kv8);
  if (workspace_bytes < L.total)
    return set_error(PKV_ERR_INVALID, "paged_attention_decode_shared: workspace of %zu bytes, %zu needed",
                     workspace_bytes, L.total);

  const unsigned char* pl = static_cast<const unsigned char*>(plan);
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  int32_t* count = reinterpret_cast<int32_t*>(ws + L.off_count);
  int32_t* v_lens = reinterpret_cast<int32_t*>(ws + L.off_lens);
  int32_t* v_offset = reinterpret_cast<int32_t*>(ws + L.off_offset);
  float* seg_o = reinterpret_cast<float*>(ws + L.off_seg_o);
  float2* seg_ml = reinterpret_cast<float2*>(ws + L.off_seg_ml);
  unsigned char* dws = ws + L.off_decode;
  const int4* entries = reinterpret_cast<const int4*>(pl + in.off_entries);
  const int4* parts = reinterpret_cast<const int4*>(pl + in.off_parts);
  const int32_t* row_start = reinterpret_cast<const int32_t*>(pl + in.off_row_start);
  const int32_t* row_ids = reinterpret_cast<const int32_t*>(pl + in.off_row_ids);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // ---- check the plan against the call
  sp::SetupArgs sa{};
  sa.entries = entries;
  sa.parts = parts;
  sa.suffix_lens = reinterpret_cast<const int32_t*>(pl + in.off_suffix_lens);
  sa.block_offset = reinterpret_cast<const int32_t*>(pl + in.off_block_offset);
  sa.row_start = row_start;
  sa.row_ids = row_ids;
  sa.context_lens = context_lens;
  sa.count = count;
  sa.v_lens = v_lens;
  sa.v_offset = v_offset;
  sa.status = status;
  sa.num_seqs = num_seqs;
  sa.num_entries = in.num_entries;
  sa.num_parts = in.num_parts;
  sa.num_partials = in.num_partials;
  sa.max_blocks = max_blocks_per_seq;
  sa.block_size = block_size;
  sa.tile_rows = 128 / group;
  sa.max_suffix_len = in.max_suffix_len;
  sa.scratch_blocks = kv8 ? L.scratch_blocks : -1;
  sp::shared_setup_kernel<<<1, sp::kSetupThreads, 0, s>>>(sa);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "shared setup launch: %s", cudaGetErrorString(e));

  // ---- shared phase, on the side stream
  int dev = 0;
  cudaError_t de = cudaGetDevice(&dev);
  if (de != cudaSuccess) return set_error(PKV_ERR_CUDA, "shared decode: cudaGetDevice: %s", cudaGetErrorString(de));
  if (dev < 0 || dev >= kMaxDevices) return set_error(PKV_ERR_INVALID, "shared decode: device %d out of range", dev);
  sp::Side side{};
  if (in.num_entries > 0) {
    const int st = sp::side_for(dev, &side);
    if (st != 0)
      return set_error(PKV_ERR_CUDA, "shared decode: side stream: %s", cudaGetErrorString(static_cast<cudaError_t>(st)));
  }
  std::unique_lock<std::mutex> lock(sp::g_side_mutex[dev], std::defer_lock);
  if (in.num_entries > 0) {
    lock.lock();
    e = cudaEventRecord(side.fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side.stream, side.fork, 0);
    if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "shared decode: fork: %s", cudaGetErrorString(e));
    SegmentLaunch sl{};
    sl.query = query;
    sl.key_cache = key_cache;
    sl.value_cache = value_cache;
    sl.block_tables = block_tables;
    int seg_blocks = num_blocks;
    if (kv8) {
      // the parts' blocks widened into the scratch pools, on the side stream before the shared phase
      sp::ScratchArgs sc{};
      sc.parts = parts;
      sc.block_tables = block_tables;
      sc.key8 = static_cast<const uint8_t*>(key_cache);
      sc.value8 = static_cast<const uint8_t*>(value_cache);
      sc.key_s = reinterpret_cast<__nv_bfloat16*>(ws + L.off_scr_k);
      sc.value_s = reinterpret_cast<__nv_bfloat16*>(ws + L.off_scr_v);
      sc.table_s = reinterpret_cast<int32_t*>(ws + L.off_scr_tab);
      sc.bad = count + 2;
      sc.status = status;
      sc.num_parts = in.num_parts;
      sc.num_seqs = num_seqs;
      sc.max_blocks = max_blocks_per_seq;
      sc.block_size = block_size;
      sc.num_blocks = num_blocks;
      sc.num_kv_heads = num_kv_heads;
      sc.scratch_blocks = L.scratch_blocks;
      if (in.num_parts > 0) {
        sp::scratch_fill_kernel<<<dim3(in.num_parts, num_kv_heads, sp::kScratchSplit), sp::kScratchThreads, 0,
                                  side.stream>>>(sc);
        e = cudaGetLastError();
        if (e != cudaSuccess) {
          cudaEventRecord(side.join, side.stream);
          cudaStreamWaitEvent(s, side.join, 0);  // leave the caller's stream joined
          return set_error(PKV_ERR_CUDA, "shared decode: scratch launch: %s", cudaGetErrorString(e));
        }
      }
      sl.key_cache = sc.key_s;
      sl.value_cache = sc.value_s;
      sl.block_tables = sc.table_s;
      sl.k_scale = k_scale;
      sl.v_scale = v_scale;
      seg_blocks = static_cast<int>(L.scratch_blocks);
    }
    sl.plan_count = count;
    sl.entries = entries;
    sl.parts = parts;
    sl.part_o = seg_o;
    sl.part_ml = seg_ml;
    sl.status = status;
    sl.num_entries = in.num_entries;
    sl.max_blocks = max_blocks_per_seq;
    sl.num_seqs = num_seqs;
    sl.num_heads = num_heads;
    sl.num_kv_heads = num_kv_heads;
    sl.block_size = block_size;
    sl.num_blocks = seg_blocks;
    sl.scale = scale;
    int rc = launch_prefill_segments(sl, side.stream);
    e = cudaEventRecord(side.join, side.stream);
    if (rc == PKV_OK && e != cudaSuccess) rc = set_error(PKV_ERR_CUDA, "shared decode: join: %s", cudaGetErrorString(e));
    if (rc != PKV_OK) {
      cudaStreamWaitEvent(s, side.join, 0);  // leave the caller's stream joined
      return rc;
    }
  }

  // ---- private phase: the remainders through the tensor-core decode, partials only
  DecodeArgs a{};
  a.out = out;
  a.query = static_cast<const __nv_bfloat16*>(query);
  if (kv8) {
    a.key_cache8 = static_cast<const uint8_t*>(key_cache);
    a.value_cache8 = static_cast<const uint8_t*>(value_cache);
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.q_split = dws + L.dec.off_qsplit;
    a.q_inv = reinterpret_cast<float*>(dws + L.dec.off_qinv);
  } else {
    a.key_cache = static_cast<const __nv_bfloat16*>(key_cache);
    a.value_cache = static_cast<const __nv_bfloat16*>(value_cache);
  }
  a.block_tables = block_tables;
  a.plan_count = reinterpret_cast<const int32_t*>(dws + L.dec.off_count);
  a.entries = reinterpret_cast<const PlanEntry*>(dws + L.dec.off_entries);
  a.arrive = reinterpret_cast<int32_t*>(dws + L.dec.off_arrive);
  a.part_o = reinterpret_cast<float*>(dws + L.dec.off_part_o);
  a.part_ml = reinterpret_cast<float2*>(dws + L.dec.off_part_ml);
  a.status = status;
  a.context_lens = v_lens;
  a.max_context_len = in.max_suffix_len;
  a.max_blocks = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.group = group;
  a.partition = L.partition;
  a.max_parts = L.dec.max_parts;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.block_offset = v_offset;
  a.always_partial = 1;
  int rc = launch_decode_plan(a, v_lens, in.max_suffix_len, s);
  if (rc == PKV_OK)
    rc = L.private_simt ? launch_decode_simt(a, head_dim, out_dtype == PKV_DTYPE_F32, s)
         : kv8          ? launch_decode_tensor_fp8(a, head_dim, out_dtype == PKV_DTYPE_F32, s)
                        : launch_decode_tensor(a, head_dim, out_dtype == PKV_DTYPE_F32, s);
  if (in.num_entries > 0) {
    e = cudaStreamWaitEvent(s, side.join, 0);  // the merge reads the shared partials
    if (rc == PKV_OK && e != cudaSuccess) rc = set_error(PKV_ERR_CUDA, "shared decode: join: %s", cudaGetErrorString(e));
  }
  if (rc != PKV_OK) return rc;

  // ---- merge
  sp::MergeArgs m{};
  m.out = out;
  m.dec_o = a.part_o;
  m.dec_ml = a.part_ml;
  m.seg_o = seg_o;
  m.seg_ml = seg_ml;
  m.v_lens = v_lens;
  m.row_start = row_start;
  m.row_ids = row_ids;
  m.bad = count + 2;
  m.num_seqs = num_seqs;
  m.num_heads = num_heads;
  m.partition = L.partition;
  m.max_parts = L.dec.max_parts;
  const int64_t units = static_cast<int64_t>(num_seqs) * num_heads;
  const unsigned grid = static_cast<unsigned>((units + sp::kMergeWarps - 1) / sp::kMergeWarps);
  if (out_dtype == PKV_DTYPE_F32)
    sp::shared_merge_kernel<true><<<grid, sp::kMergeWarps * 32, 0, s>>>(m);
  else
    sp::shared_merge_kernel<false><<<grid, sp::kMergeWarps * 32, 0, s>>>(m);
  e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "shared merge launch: %s", cudaGetErrorString(e));
  return PKV_OK;
}

extern "C" int pkv_paged_attention_decode_shared(void* out, int out_dtype, const void* query, const void* key_cache,
                                                 const void* value_cache, const int32_t* block_tables,
                                                 int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                                                 int num_heads, int num_kv_heads, int head_dim, int block_size,
                                                 int num_blocks, float scale, const void* plan,
                                                 const pkv_shared_plan_info* info, void* workspace,
                                                 size_t workspace_bytes, int32_t* status, pkv_stream_t stream) {
  clear_error();
  return shared_impl(false, out, out_dtype, query, key_cache, value_cache, nullptr, nullptr, block_tables,
                     max_blocks_per_seq, context_lens, num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                     num_blocks, scale, plan, info, workspace, workspace_bytes, status, stream);
}

extern "C" int pkv_paged_attention_decode_shared_fp8(void* out, int out_dtype, const void* query,
                                                     const void* key_cache, const void* value_cache,
                                                     const float* k_scale, const float* v_scale,
                                                     const int32_t* block_tables, int max_blocks_per_seq,
                                                     const int32_t* context_lens, int num_seqs, int num_heads,
                                                     int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                                     float scale, const void* plan, const pkv_shared_plan_info* info,
                                                     void* workspace, size_t workspace_bytes, int32_t* status,
                                                     pkv_stream_t stream) {
  clear_error();
  return shared_impl(true, out, out_dtype, query, key_cache, value_cache, k_scale, v_scale, block_tables,
                     max_blocks_per_seq, context_lens, num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                     num_blocks, scale, plan, info, workspace, workspace_bytes, status, stream);
}
