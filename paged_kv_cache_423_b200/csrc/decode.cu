// Paged decode attention: the work plan, the CUDA-core streaming kernel and the
// C-ABI entry points.
//
// What is computed (intelliparadigm article "PagedAttention：操作系统分页思想的跨界创新",
// §2.1, paged_attention pseudo-code): for each sequence and query head, the logical
// block of token t is t // block_size, the block table gives its physical block,
// K and V are read from there, and the output is softmax(scale * q·Kᵀ)·V over the
// sequence's context.  §2.1 also states the kernel idea this file keeps: splice the
// non-contiguous pages on the fly through shared memory, with prefetch.
//
// How it maps to sm_100a:
//   * plan kernel (one CTA): splits every sequence into partitions of at most
//     `partition` tokens and counting-sorts the (sequence, partition) entries by
//     length, longest first, so the persistent kernel hands out big items first and
//     fills the tail with small ones.
//   * streaming kernel (persistent, CUDA cores): every warp is an independent
//     consumer with its own ring of shared-memory stages.  Lane 0 streams 16-token
//     slices of (block, kv head) tiles into the ring with 1-D bulk copies (TMA
//     engine, mbarrier completion), several stages ahead of the math, and runs ahead
//     across item boundaries (block-table slices of the next item are prefetched one
//     item early).  Scores use a transposed warp reduction (one shuffle per token),
//     the softmax is online in fp32 and base 2, P·V accumulates in fp32 registers.
//   * split partitions write an unnormalised partial (o, m, l); the last partition
//     of a (sequence, head) to arrive (device-scope atomic counter) merges all
//     partials by log-sum-exp rescaling and writes the output, so there is no
//     separate reduce launch.  No thread ever waits for another CTA.
#include <cuda_runtime.h>

#include <algorithm>
#include <type_traits>

#include "decode_common.cuh"
#include "launch_setup.cuh"
#include "pkv_internal.h"

// Warps per CTA, ring stages per warp, and dynamic (counter) instead of static
// work distribution of the CUDA-core kernel; compile-time overridable for sweeps.
#ifndef PKV_SIMT_WARPS
#define PKV_SIMT_WARPS 4
#endif
#ifndef PKV_SIMT_STAGES
#define PKV_SIMT_STAGES 2
#endif
#ifndef PKV_SIMT_DYNAMIC
#define PKV_SIMT_DYNAMIC 1
#endif
// Ring stages per warp for an 8-bit pool (32-token stages of the same 8 KiB).
#ifndef PKV_SIMT_STAGES8
#define PKV_SIMT_STAGES8 2
#endif

namespace pkv {

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------------------
// Plan kernel
// ---------------------------------------------------------------------------

constexpr int kPlanThreads = 1024;

// Bucket of an entry of `ntok` tokens: longest first, 513 buckets whatever the
// split size (exact for splits up to 512 tokens, coarser beyond).
__device__ __forceinline__ int plan_bucket(int ntok, int partition) {
  return static_cast<int>((static_cast<int64_t>(partition - ntok) * (kPlanBuckets - 1)) / partition);
}

__global__ void __launch_bounds__(kPlanThreads)
    plan_kernel(const int32_t* __restrict__ context_lens, int num_seqs, int max_context_len, int max_table_tokens,
                int partition, PlanEntry* __restrict__ entries, int32_t* __restrict__ plan_count,
                int32_t* __restrict__ arrive, int n_arrive, int32_t* status) {
  __shared__ int bucket[kPlanBuckets];
  __shared__ int warp_total[32];
  griddep_launch_dependents();  // the decode kernel may be scheduled now; it waits for this one to end
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kPlanBuckets; i += blockDim.x) bucket[i] = 0;
  for (int i = tid; i < n_arrive; i += blockDim.x) arrive[i] = 0;
  __syncthreads();
  // One thread per sequence.  Its full-length partitions all fall in bucket 0 and
  // only the last may be shorter, so a sequence costs at most two atomics.
  for (int s = tid; s < num_seqs; s += blockDim.x) {
    int L = context_lens[s];
    if (L < 0 || L > max_context_len || L > max_table_tokens) {
      set_status(status, PKV_DEV_BAD_CONTEXT);
      L = 0;
    }
    const int full = L / partition;
    const int tail = L - full * partition;
    if (full > 0) atomicAdd(&bucket[0], full);
    if (tail > 0 || L == 0) atomicAdd(&bucket[plan_bucket(tail, partition)], 1);
  }
  __syncthreads();
  // Exclusive scan of the bucket counts (513 buckets <= 1024 threads).
  const int v = tid < kPlanBuckets ? bucket[tid] : 0;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_total[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (blockDim.x >> 5) ? warp_total[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, w, o);
      if (lane >= o) w += y;
    }
    warp_total[lane] = w;
  }
  __syncthreads();
  const int excl = x - v + (warp > 0 ? warp_total[warp - 1] : 0);
  __syncthreads();
  if (tid < kPlanBuckets) bucket[tid] = excl;
  if (tid == 0) {
    plan_count[0] = warp_total[31];
    plan_count[1] = 0;  // work-item counter of the tensor-core kernel
  }
  __syncthreads();
  for (int s = tid; s < num_seqs; s += blockDim.x) {
    int L = context_lens[s];
    if (L < 0 || L > max_context_len || L > max_table_tokens) L = 0;
    const int full = L / partition;
    const int tail = L - full * partition;
    const int np = L == 0 ? 1 : full + (tail > 0);
    if (full > 0) {
      const int pos = atomicAdd(&bucket[0], full);
      for (int p = 0; p < full; ++p) entries[pos + p] = make_int4(s, p, np, L);
    }
    if (tail > 0 || L == 0) {
      const int pos = atomicAdd(&bucket[plan_bucket(tail, partition)], 1);
      entries[pos] = make_int4(s, full, np, L);
    }
  }
}

// ---------------------------------------------------------------------------
// CUDA-core streaming kernel
// ---------------------------------------------------------------------------

// Tokens per ring stage: 16-row slices for bf16 (4 KiB of K at D = 128); an 8-bit
// pool takes 32 tokens per stage, so a stage still moves 8 KiB of K and V and the
// fixed cost of a stage (wait, reductions, softmax) is spread over as many bytes.
template <bool KV8>
constexpr int stage_tokens() { return KV8 ? 2 * kStageTokens : kStageTokens; }
// Values per lane of the 8-bit pool's P·V accumulators (a 16-byte chunk of a head_dim-128 row).
constexpr int kPV8 = 16;

template <int D, int STAGES, bool KV8 = false>
struct __align__(128) WarpRing {
  using KvT = std::conditional_t<KV8, uint8_t, __nv_bfloat16>;  // bf16 or e4m3 pool elements
  static constexpr int ST = stage_tokens<KV8>();
  KvT k[STAGES][ST * D];
  KvT v[STAGES][ST * D];
  __nv_bfloat16 q[STAGES][D];
  float2 p[ST];  // (p_t, p_t) of the stage being consumed, read back as packed pairs
                 // (8-bit pool: p_t rounded to f16, packed as 32 halves in the first 64 bytes)
  uint64_t full[STAGES];
  int4 meta[STAGES];  // x seq, y query head, z part | nparts << 16, w n_valid | flags (first, last, q present)
};

// Per-item state of the issuing side (warp-uniform except `table`).
struct IssueItem {
  int64_t id;      // item index, or -1 when there is none
  PlanEntry e;     // seq, part, nparts, L
  int table;       // lane j: physical block of the item's j-th block (prefetched)
};

__device__ __forceinline__ int item_stages(const PlanEntry& e, int partition, int stage_tok) {
  const int ntok = e.w == 0 ? 0 : min(partition, e.w - e.y * partition);
  return ntok == 0 ? 1 : (ntok + stage_tok - 1) / stage_tok;
}

// Load lane j's table entry for the item (block tok0/bs + j, from the row's block_offset on
// when there is one), 0 past the item.
__device__ __forceinline__ int load_item_table(const DecodeArgs& a, const PlanEntry& e, int lane) {
  const int tok0 = e.y * a.partition;
  const int ntok = e.w == 0 ? 0 : min(a.partition, e.w - tok0);
  const int nblk = (ntok + a.block_size - 1) / a.block_size;
  if (lane >= nblk) return 0;
  const int off = a.block_offset ? __ldg(a.block_offset + e.x) : 0;
  return __ldg(a.block_tables + static_cast<int64_t>(e.x) * a.max_blocks + tok0 / a.block_size + off + lane);
}

// a0 += q.lo * k.lo, a1 += q.hi * k.hi with bf16 operands and fp32 accumulation
// (sm_100 mixed-precision FMA; the bf16 x bf16 product is exact in fp32).
__device__ __forceinline__ void dot_bf16x2(float& a0, float& a1, uint32_t q, uint32_t k) {
  asm("{\n\t.reg .b16 ql, qh, kl, kh;\n\t"
      "mov.b32 {ql, qh}, %2;\n\t"
      "mov.b32 {kl, kh}, %3;\n\t"
      "fma.rn.f32.bf16 %0, ql, kl, %0;\n\t"
      "fma.rn.f32.bf16 %1, qh, kh, %1;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(q), "r"(k));
}

template <int D, bool OUT_F32>
__device__ __forceinline__ void store_row(const DecodeArgs& a, int seq, int qh, int col, const float* o,
                                          float inv) {
  constexpr int EPL = D / 32;
  const int64_t base = (static_cast<int64_t>(seq) * a.num_heads + qh) * D + col;
  if constexpr (OUT_F32) {
    float* out = static_cast<float*>(a.out) + base;
    if constexpr (EPL == 4)
      *reinterpret_cast<float4*>(out) = make_float4(o[0] * inv, o[1] * inv, o[2] * inv, o[3] * inv);
    else
      *reinterpret_cast<float2*>(out) = make_float2(o[0] * inv, o[1] * inv);
  } else {
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + base;
    if constexpr (EPL == 4)
      *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16x2(o[0] * inv, o[1] * inv), pack_bf16x2(o[2] * inv, o[3] * inv));
    else
      *reinterpret_cast<uint32_t*>(out) = pack_bf16x2(o[0] * inv, o[1] * inv);
  }
}

// Lane roles inside a warp.
//   q·K: two lanes per row, each over half of head_dim (64 or 32 values, NC 16-byte
//        chunks).  Lane k of a row visits its chunks in the rotated order
//        (k + i) mod NC, so the 8 lanes of each shared-memory phase always hit 8
//        different 16-byte bank groups although every row starts at bank 0.
//   P·V: lane l owns head_dim/32 consecutive output values of every row.
template <int D, bool KV8 = false>
struct LaneMap {
  static constexpr int NC = D / 16;                  // 16-byte chunks per half row
  static constexpr int PARTNER = D == 128 ? 16 : 4;  // the lane holding the other half of the row
  __device__ static int row(int lane) { return D == 128 ? (lane & 15) : ((lane & 3) | ((lane >> 3) << 2)); }
  __device__ static int half(int lane) { return D == 128 ? (lane >> 4) : ((lane >> 2) & 1); }
  __device__ static float max_rows(float x) {  // max over the 16 rows (lanes with the same half)
    constexpr int m0 = 1, m1 = 2, m2 = D == 128 ? 4 : 8, m3 = D == 128 ? 8 : 16;
    x = fmaxf(x, __shfl_xor_sync(kFull, x, m0));
    x = fmaxf(x, __shfl_xor_sync(kFull, x, m1));
    x = fmaxf(x, __shfl_xor_sync(kFull, x, m2));
    return fmaxf(x, __shfl_xor_sync(kFull, x, m3));
  }
};

// 8-bit pool, head_dim 128: a K row is 128 bytes, a half row 64 bytes = 4 chunks.
// The two halves of a row sit in adjacent lanes (row = lane / 2), so each group of 8
// lanes covers 4 rows x both halves and, with the rotated chunk order, 8 different
// 16-byte bank groups.
template <>
struct LaneMap<128, true> {
  static constexpr int NC = 4;
  static constexpr int PARTNER = 1;
  __device__ static int row(int lane) { return lane >> 1; }
  __device__ static int half(int lane) { return lane & 1; }
  __device__ static float max_rows(float x) {
    x = fmaxf(x, __shfl_xor_sync(kFull, x, 2));
    x = fmaxf(x, __shfl_xor_sync(kFull, x, 4));
    x = fmaxf(x, __shfl_xor_sync(kFull, x, 8));
    return fmaxf(x, __shfl_xor_sync(kFull, x, 16));
  }
};

// ---- e4m3 helpers (8-bit pool)
// Four e4m3 codes of a word (low byte first) -> two f16x2 (bytes 0,1 and 2,3), exactly
// (every e4m3 value is an f16 value).
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}
// a0 += x.lo * y.lo, a1 += x.hi * y.hi with f16 operands and fp32 accumulation
// (sm_100 mixed-precision FMA; the f16 x f16 product is exact in fp32).
__device__ __forceinline__ void dot_f16x2(float& a0, float& a1, uint32_t x, uint32_t y) {
  asm("{\n\t.reg .b16 xl, xh, yl, yh;\n\t"
      "mov.b32 {xl, xh}, %2;\n\t"
      "mov.b32 {yl, yh}, %3;\n\t"
      "fma.rn.f32.f16 %0, xl, yl, %0;\n\t"
      "fma.rn.f32.f16 %1, xh, yh, %1;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(x), "r"(y));
}
// a += p * x.lo, b += p * x.hi with p the low (HI = false) or high f16 of `p16`
template <bool HI>
__device__ __forceinline__ void axpy_f16x2(float& a, float& b, uint32_t p16, uint32_t x) {
  if constexpr (HI)
    asm("{\n\t.reg .b16 pl, ph, xl, xh;\n\t"
        "mov.b32 {pl, ph}, %2;\n\t"
        "mov.b32 {xl, xh}, %3;\n\t"
        "fma.rn.f32.f16 %0, ph, xl, %0;\n\t"
        "fma.rn.f32.f16 %1, ph, xh, %1;\n\t}"
        : "+f"(a), "+f"(b)
        : "r"(p16), "r"(x));
  else
    asm("{\n\t.reg .b16 pl, ph, xl, xh;\n\t"
        "mov.b32 {pl, ph}, %2;\n\t"
        "mov.b32 {xl, xh}, %3;\n\t"
        "fma.rn.f32.f16 %0, pl, xl, %0;\n\t"
        "fma.rn.f32.f16 %1, pl, xh, %1;\n\t}"
        : "+f"(a), "+f"(b)
        : "r"(p16), "r"(x));
}
__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float f16lo_to_f32(uint32_t w) {
  float r;
  asm("{\n\t.reg .b16 lo;\n\tcvt.u16.u32 lo, %1;\n\tcvt.f32.f16 %0, lo;\n\t}" : "=f"(r) : "r"(w));
  return r;
}

template <int D, bool OUT_F32, int WARPS, int STAGES, bool KV8 = false>
__global__ void __launch_bounds__(WARPS * 32) decode_simt_kernel(const __grid_constant__ DecodeArgs a) {
  static_assert(!KV8 || D == 128, "the 8-bit pool path is head_dim 128");
  constexpr int EPL = D / 32;                                  // output values per lane: 2 or 4
  constexpr int NPAIR = EPL / 2;                               // packed fp32 pairs per lane
  constexpr int NC = LaneMap<D, KV8>::NC;
  using Ring = WarpRing<D, STAGES, KV8>;
  constexpr int ST = Ring::ST;
  constexpr uint32_t kKVBytes = ST * D * sizeof(typename Ring::KvT);          // a full stage of K (or V)
  constexpr uint32_t kSliceBytes = kStageTokens * D * sizeof(typename Ring::KvT);  // one 16-row slice
  constexpr uint32_t kQBytes = D * sizeof(__nv_bfloat16);
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Ring& ring = reinterpret_cast<Ring*>(smem_raw)[warp];
  const int qk_row = LaneMap<D, KV8>::row(lane), qk_half = LaneMap<D, KV8>::half(lane);

  griddep_wait();  // the plan kernel before this one has finished
  const int64_t n_items = static_cast<int64_t>(a.plan_count[0]) * a.num_heads;
  // Work distribution over the plan (longest items first): every warp starts with
  // items w and w + #warps; after that it takes the next unclaimed item from a
  // global counter, so warps that finish early do more of the tail.
  const int64_t stride = static_cast<int64_t>(gridDim.x) * WARPS;
  const int64_t first_item = static_cast<int64_t>(blockIdx.x) * WARPS + warp;
#if PKV_SIMT_DYNAMIC
  int* work_counter = const_cast<int*>(a.plan_count) + 1;
  auto take = [&]() -> int64_t {
    int v = 0;
    if (lane == 0) v = atomicAdd(work_counter, 1);
    return 2 * stride + __shfl_sync(kFull, v, 0);
  };
#endif
  if (first_item >= n_items) return;

  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < STAGES; ++s) mbar_init(&ring.full[s], 1);
    fence_barrier_init();
  }
  __syncwarp();
  const uint64_t policy = l2_policy_kv();

  // ---- issuing side: current item, next item (table prefetched), item after (entry prefetched)
  auto entry_of = [&](int64_t id) -> PlanEntry {
    return id < n_items ? a.entries[id / a.num_heads] : make_int4(0, 0, 0, 0);
  };
  IssueItem cur, nxt;
  PlanEntry nx2_e;
  int64_t nx2_id;
  cur.id = first_item;
  cur.e = entry_of(cur.id);
  cur.table = load_item_table(a, cur.e, lane);
  nxt.id = first_item + stride < n_items ? first_item + stride : -1;
  nxt.e = entry_of(first_item + stride);
#if PKV_SIMT_DYNAMIC
  {
    const int64_t i2 = nxt.id >= 0 ? take() : n_items;
    nx2_id = i2 < n_items ? i2 : -1;
    nx2_e = entry_of(i2);
  }
#else
  nx2_id = first_item + 2 * stride < n_items ? first_item + 2 * stride : -1;
  nx2_e = entry_of(first_item + 2 * stride);
#endif
  nxt.table = nxt.id >= 0 ? load_item_table(a, nxt.e, lane) : 0;
  int cur_stage = 0;
  int cur_nstages = item_stages(cur.e, a.partition, ST);
  bool issue_done = false;

  // Issue the next stage into `slot`; false when every item has been issued.
  auto issue = [&](int slot) -> bool {
    if (issue_done) return false;
    if (cur_stage == cur_nstages) {
      if (nxt.id < 0) {
        issue_done = true;
        return false;
      }
      cur = nxt;
      nxt.id = nx2_id;
      nxt.e = nx2_e;
      nxt.table = nxt.id >= 0 ? load_item_table(a, nxt.e, lane) : 0;
#if PKV_SIMT_DYNAMIC
      if (nx2_id >= 0) {
        const int64_t i2 = take();
        nx2_id = i2 < n_items ? i2 : -1;
      }
#else
      nx2_id = nx2_id >= 0 && nx2_id + stride < n_items ? nx2_id + stride : -1;
#endif
      nx2_e = entry_of(nx2_id >= 0 ? nx2_id : n_items);
      cur_stage = 0;
      cur_nstages = item_stages(cur.e, a.partition, ST);
    }
    const PlanEntry e = cur.e;
    const int qh = static_cast<int>(cur.id % a.num_heads);
    const int kvh = qh / a.group;
    const int local_tok = cur_stage * ST;
    const int tok = e.y * a.partition + local_tok;                       // first token of the stage
    const int n_tok = e.w == 0 ? 0 : min(ST, e.w - tok);
    const int phys = __shfl_sync(kFull, cur.table, local_tok / a.block_size);
    // 8-bit pool: the stage's second 16-row slice (maybe in the next block at bs 16)
    const int phys2 = KV8 ? __shfl_sync(kFull, cur.table, (local_tok + kStageTokens) / a.block_size) : 0;
    const bool two = KV8 && n_tok > kStageTokens;
    const bool ok = n_tok > 0 && phys >= 0 && phys < a.num_blocks && (!two || (phys2 >= 0 && phys2 < a.num_blocks));
    const bool first = cur_stage == 0, last = cur_stage == cur_nstages - 1;
    const bool with_q = first && n_tok > 0;
    if (lane == 0) {
      if (n_tok > 0 && !ok) set_status(a.status, PKV_DEV_BAD_BLOCK);
      ring.meta[slot] = make_int4(e.x, qh, e.y | (e.z << 16),
                                  (ok ? n_tok : 0) | (first ? 0x100 : 0) | (last ? 0x200 : 0) | (with_q ? 0x400 : 0));
      const uint32_t kv_bytes = KV8 ? (two ? 2 : 1) * 2 * kSliceBytes : 2 * kKVBytes;
      const uint32_t bytes = (ok ? kv_bytes : 0) + (with_q ? kQBytes : 0);
      mbar_arrive_expect_tx(&ring.full[slot], bytes);
      if (with_q)
        bulk_copy_g2s(ring.q[slot], a.query + (static_cast<int64_t>(e.x) * a.num_heads + qh) * D, kQBytes,
                      &ring.full[slot], policy);
      if (ok) {
        const int64_t row = (static_cast<int64_t>(phys) * a.num_kv_heads + kvh) * a.block_size + local_tok % a.block_size;
        if constexpr (KV8) {
          bulk_copy_g2s(ring.k[slot], a.key_cache8 + row * D, kSliceBytes, &ring.full[slot], policy);
          bulk_copy_g2s(ring.v[slot], a.value_cache8 + row * D, kSliceBytes, &ring.full[slot], policy);
          if (two) {
            const int t2 = local_tok + kStageTokens;
            const int64_t row2 =
                (static_cast<int64_t>(phys2) * a.num_kv_heads + kvh) * a.block_size + t2 % a.block_size;
            bulk_copy_g2s(ring.k[slot] + kStageTokens * D, a.key_cache8 + row2 * D, kSliceBytes, &ring.full[slot],
                          policy);
            bulk_copy_g2s(ring.v[slot] + kStageTokens * D, a.value_cache8 + row2 * D, kSliceBytes,
                          &ring.full[slot], policy);
          }
        } else {
          bulk_copy_g2s(ring.k[slot], a.key_cache + row * D, kKVBytes, &ring.full[slot], policy);
          bulk_copy_g2s(ring.v[slot], a.value_cache + row * D, kKVBytes, &ring.full[slot], policy);
        }
      }
    }
    ++cur_stage;
    return true;
  };

  // ---- consuming side
  // this lane's half of q in rotated chunk order: raw bf16 pairs, or (8-bit pool)
  // f16 pairs, two uint4 per 16-code chunk
  constexpr int NQ = KV8 ? 2 * NC : NC;
  uint4 qv[NQ];
  uint64_t o[NPAIR];            // packed fp32 output accumulators
  // 8-bit pool: fp32 accumulators of the lane's 16 values (a 16-byte chunk of a row) over the
  // rows of its row group; the four row groups are added once per item
  float o8[KV8 ? kPV8 : 1];
  float score_scale = a.scale_log2, out_scale = 1.f;
  float m = -INFINITY, lsum = 0.f;
#pragma unroll
  for (int i = 0; i < NQ; ++i) qv[i] = make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int j = 0; j < (KV8 ? kPV8 : 1); ++j) o8[j] = 0.f;
#pragma unroll
  for (int j = 0; j < NPAIR; ++j) o[j] = f2pack(0.f, 0.f);

  int issued = 0;
  for (int s = 0; s < STAGES; ++s) {
    if (!issue(s)) break;
    ++issued;
  }
  int consumed = 0;
  bool timed_out = false;
  while (consumed < issued) {
    const int slot = consumed % STAGES;
    if (!__all_sync(kFull, pipe_wait(&ring.full[slot], (consumed / STAGES) & 1))) {  // warp-uniform
      timed_out = true;
      break;
    }
    const int4 mt = ring.meta[slot];
    const int n_valid = mt.w & 0xff;
    const bool first = mt.w & 0x100, last = mt.w & 0x200;
    if (first) {
      m = -INFINITY;
      lsum = 0.f;
#pragma unroll
      for (int j = 0; j < NPAIR; ++j) o[j] = f2pack(0.f, 0.f);
      if constexpr (KV8) {
#pragma unroll
        for (int j = 0; j < kPV8; ++j) o8[j] = 0.f;
        if (mt.w & 0x400) {
          // q to f16 for the mixed-precision products.  bf16 values of magnitude
          // >= 2^15 would overflow f16: then the whole vector is scaled by 2^-16
          // (and the score scale by 2^16).
          const uint4* qs = reinterpret_cast<const uint4*>(ring.q[slot]);
          bool big = false;
#pragma unroll
          for (int i = 0; i < NC; ++i) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint4 w = qs[qk_half * 2 * NC + 2 * ((i + qk_row) & (NC - 1)) + h];
              const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int c = 0; c < 4; ++c)
                big |= fabsf(bf16lo(ws[c])) >= 32768.f || fabsf(bf16hi(ws[c])) >= 32768.f;
            }
          }
          const float qscale = __any_sync(kFull, big) ? 1.f / 65536.f : 1.f;
#pragma unroll
          for (int i = 0; i < NC; ++i) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint4 w = qs[qk_half * 2 * NC + 2 * ((i + qk_row) & (NC - 1)) + h];
              qv[2 * i + h] = make_uint4(f32x2_to_f16x2(bf16lo(w.x) * qscale, bf16hi(w.x) * qscale),
                                         f32x2_to_f16x2(bf16lo(w.y) * qscale, bf16hi(w.y) * qscale),
                                         f32x2_to_f16x2(bf16lo(w.z) * qscale, bf16hi(w.z) * qscale),
                                         f32x2_to_f16x2(bf16lo(w.w) * qscale, bf16hi(w.w) * qscale));
            }
          }
          const int kvh = mt.y / a.group;
          score_scale = a.scale_log2 * __ldg(a.k_scale + kvh) / qscale;
          out_scale = __ldg(a.v_scale + kvh);
        }
      } else if (mt.w & 0x400) {
        const uint4* qs = reinterpret_cast<const uint4*>(ring.q[slot]);
#pragma unroll
        for (int i = 0; i < NC; ++i) qv[i] = qs[qk_half * NC + ((i + qk_row) & (NC - 1))];
      }
    }
    if (n_valid > 0) {
      float alpha;
      if constexpr (KV8) {
        // ---- scores, 8-bit pool: rows r and r + 16 of the 32-token stage; two lanes per
        // row, f16 x e4m3 products accumulated in fp32
        float sc[2];
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
          const int r = qk_row + pass * kStageTokens;
          const uint4* krow = reinterpret_cast<const uint4*>(ring.k[slot] + r * D) + qk_half * NC;
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f, b0 = 0.f, b1 = 0.f, b2 = 0.f, b3 = 0.f;
#pragma unroll
          for (int i = 0; i < NC; ++i) {
            const uint4 kw = krow[(i + qk_row) & (NC - 1)];
            const uint32_t kws[4] = {kw.x, kw.y, kw.z, kw.w};
            const uint4 q0 = qv[2 * i], q1 = qv[2 * i + 1];
            const uint32_t qs[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t k01, k23;
              e4m3x4_to_f16x2x2(kws[c], k01, k23);
              if (c & 1) {
                dot_f16x2(b0, b1, qs[2 * c], k01);
                dot_f16x2(b2, b3, qs[2 * c + 1], k23);
              } else {
                dot_f16x2(a0, a1, qs[2 * c], k01);
                dot_f16x2(a2, a3, qs[2 * c + 1], k23);
              }
            }
          }
          sc[pass] = (a0 + a1) + (a2 + a3) + ((b0 + b1) + (b2 + b3));
        }
        sc[0] += __shfl_xor_sync(kFull, sc[0], LaneMap<D, KV8>::PARTNER);
        sc[1] += __shfl_xor_sync(kFull, sc[1], LaneMap<D, KV8>::PARTNER);
        const bool v0 = qk_row < n_valid, v1 = qk_row + kStageTokens < n_valid;
        const float x0 = v0 ? sc[0] * score_scale : -INFINITY;
        const float x1 = v1 ? sc[1] * score_scale : -INFINITY;
        const float m_new = fmaxf(m, LaneMap<D, KV8>::max_rows(fmaxf(x0, x1)));
        alpha = exp2f(m - m_new);
        // the weights the P·V products use: p rounded to f16; the sum adds the same values
        const uint32_t p16a = f32x2_to_f16x2(v0 ? exp2f(x0 - m_new) : 0.f, 0.f);
        const uint32_t p16b = f32x2_to_f16x2(v1 ? exp2f(x1 - m_new) : 0.f, 0.f);
        m = m_new;
        lsum = fmaf(lsum, alpha, f16lo_to_f32(p16a) + f16lo_to_f32(p16b));
        if (qk_half == 0) {
          uint16_t* p16 = reinterpret_cast<uint16_t*>(ring.p);
          p16[qk_row] = static_cast<uint16_t>(p16a);
          p16[qk_row + kStageTokens] = static_cast<uint16_t>(p16b);
        }
      } else {
      // ---- scores: two lanes per row, bf16 x bf16 products accumulated in fp32
      const uint4* krow = reinterpret_cast<const uint4*>(ring.k[slot] + qk_row * D) + qk_half * NC;
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
      for (int i = 0; i < NC; ++i) {
        const uint4 kw = krow[(i + qk_row) & (NC - 1)];
        dot_bf16x2(a0, a1, qv[i].x, kw.x);
        dot_bf16x2(a2, a3, qv[i].y, kw.y);
        dot_bf16x2(a0, a1, qv[i].z, kw.z);
        dot_bf16x2(a2, a3, qv[i].w, kw.w);
      }
      float sc = (a0 + a1) + (a2 + a3);
      sc += __shfl_xor_sync(kFull, sc, LaneMap<D, KV8>::PARTNER);
      // ---- online softmax in base 2 over the stage's rows
      const bool valid = qk_row < n_valid;
      const float x = valid ? sc * score_scale : -INFINITY;
      const float m_new = fmaxf(m, LaneMap<D, KV8>::max_rows(x));
      alpha = exp2f(m - m_new);
      const float p = valid ? exp2f(x - m_new) : 0.f;
      m = m_new;
      lsum = fmaf(lsum, alpha, p);
      if (qk_half == 0) ring.p[qk_row] = make_float2(p, p);
      }
      __syncwarp();
      // ---- P·V: packed fp32 pairs, rows past n_valid never touched (stale rows may be NaN)
      if constexpr (KV8) {
        // ---- P·V over e4m3 rows: row group g = lane / 8 takes rows 8g..8g+7 of the stage and
        // lane l its 16-byte chunk l % 8 of each (16 values); f16 x f16 products, fp32 sums.
        // Rows past n_valid are not loaded (stale rows may hold NaN codes).
#pragma unroll
        for (int j = 0; j < kPV8; ++j) o8[j] *= alpha;
        const int g = lane >> 3;
        const uint8_t* vb = ring.v[slot] + g * 8 * D + (lane & 7) * 16;
        const uint4 pw = reinterpret_cast<const uint4*>(ring.p)[g];  // p of rows 8g..8g+7 (f16)
        const uint32_t pws[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          uint4 w = make_uint4(0, 0, 0, 0);
          if (g * 8 + k < n_valid) w = *reinterpret_cast<const uint4*>(vb + k * D);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t v01, v23;
            e4m3x4_to_f16x2x2(ws[c], v01, v23);
            if (k & 1) {
              axpy_f16x2<true>(o8[4 * c], o8[4 * c + 1], pws[k >> 1], v01);
              axpy_f16x2<true>(o8[4 * c + 2], o8[4 * c + 3], pws[k >> 1], v23);
            } else {
              axpy_f16x2<false>(o8[4 * c], o8[4 * c + 1], pws[k >> 1], v01);
              axpy_f16x2<false>(o8[4 * c + 2], o8[4 * c + 3], pws[k >> 1], v23);
            }
          }
        }
      } else {
      const uint64_t alpha2 = f2pack(alpha, alpha);
#pragma unroll
      for (int j = 0; j < NPAIR; ++j) o[j] = fmul2(o[j], alpha2);
      const uint64_t* pp = reinterpret_cast<const uint64_t*>(ring.p);
      const __nv_bfloat16* vb = ring.v[slot] + lane * EPL;
      if (n_valid == kStageTokens) {
#pragma unroll
        for (int t = 0; t < kStageTokens; ++t) {
          const uint64_t p2 = pp[t];
          if constexpr (EPL == 4) {
            const uint2 w = *reinterpret_cast<const uint2*>(vb + t * D);
            o[0] = ffma2(p2, bf16x2_to_f2(w.x), o[0]);
            o[1] = ffma2(p2, bf16x2_to_f2(w.y), o[1]);
          } else {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(vb + t * D);
            o[0] = ffma2(p2, bf16x2_to_f2(w), o[0]);
          }
        }
      } else {
#pragma unroll 4
        for (int t = 0; t < n_valid; ++t) {
          const uint64_t p2 = pp[t];
          if constexpr (EPL == 4) {
            const uint2 w = *reinterpret_cast<const uint2*>(vb + t * D);
            o[0] = ffma2(p2, bf16x2_to_f2(w.x), o[0]);
            o[1] = ffma2(p2, bf16x2_to_f2(w.y), o[1]);
          } else {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(vb + t * D);
            o[0] = ffma2(p2, bf16x2_to_f2(w), o[0]);
          }
        }
      }
      }  // bf16 P·V
    }
    if (last) {
      const int seq = mt.x, qh = mt.y, part = mt.z & 0xffff, nparts = mt.z >> 16;
      float of[EPL];
      // the lane's first output column: 8-bit pool, after the row groups' sums are scattered,
      // values 4g..4g+3 of its chunk
      const int col = KV8 ? (lane & 7) * 16 + (lane >> 3) * 4 : lane * EPL;
      if constexpr (KV8) {
        // Add the four row groups' sums, each lane keeping 4 of its chunk's 16 values: across
        // lanes l and l ^ 16 (groups g, g ^ 2) the halves 8 (g >> 1).. go to their owner, then
        // across l and l ^ 8 (g, g ^ 1) the quarters 4 (g & 1)...
        const bool hi = lane & 16, odd = lane & 8;
        float h8[8], q4[4];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float give = hi ? o8[j] : o8[8 + j];
          h8[j] = (hi ? o8[8 + j] : o8[j]) + __shfl_xor_sync(kFull, give, 16);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float give = odd ? h8[j] : h8[4 + j];
          q4[j] = (odd ? h8[4 + j] : h8[j]) + __shfl_xor_sync(kFull, give, 8);
        }
#pragma unroll
        for (int j = 0; j < EPL; ++j) of[j] = q4[j] * out_scale;  // the value scale of the kv head
      } else {
#pragma unroll
        for (int j = 0; j < NPAIR; ++j) {
          const float2 f = f2unpack(o[j]);
          of[2 * j] = f.x;
          of[2 * j + 1] = f.y;
        }
      }
      float l = lsum;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(kFull, l, off);
      l *= 0.5f;  // every row's weight was held by its two lanes
      if (nparts == 1 && !a.always_partial) {
        store_row<D, OUT_F32>(a, seq, qh, col, of, l > 0.f ? 1.f / l : 0.f);
      } else if (a.always_partial) {
        // every item's partial for the caller's merge (the shared-prefix decode's private phase)
        const int64_t pidx = (static_cast<int64_t>(seq) * a.num_heads + qh) * a.max_parts + part;
        float* po = a.part_o + pidx * D + col;
#pragma unroll
        for (int j = 0; j < EPL; ++j) po[j] = of[j];
        if (lane == 0) a.part_ml[pidx] = make_float2(m, l);
      } else {
        const int64_t unit = static_cast<int64_t>(seq) * a.num_heads + qh;
        const int64_t pidx = unit * a.max_parts + part;
        float* po = a.part_o + pidx * D + col;
#pragma unroll
        for (int j = 0; j < EPL; ++j) po[j] = of[j];
        if (lane == 0) a.part_ml[pidx] = make_float2(m, l);
        __threadfence();
        __syncwarp();
        int prev = 0;
        if (lane == 0) prev = atomicAdd(a.arrive + unit, 1);
        prev = __shfl_sync(kFull, prev, 0);
        if (prev == nparts - 1) {
          // Last partition in: merge every partial of this (sequence, head).
          __threadfence();
          const float2* ml = a.part_ml + unit * a.max_parts;
          float M = -INFINITY;
          for (int p = 0; p < nparts; ++p) M = fmaxf(M, __ldcg(&ml[p].x));
          float acc[EPL], Ls = 0.f;
#pragma unroll
          for (int j = 0; j < EPL; ++j) acc[j] = 0.f;
          const float* pb = a.part_o + unit * a.max_parts * D + col;
          for (int p = 0; p < nparts; ++p) {
            const float2 mlp = __ldcg(&ml[p]);
            const float w = exp2f(mlp.x - M);
            Ls = fmaf(w, mlp.y, Ls);
#pragma unroll
            for (int j = 0; j < EPL; ++j) acc[j] = fmaf(w, __ldcg(pb + static_cast<int64_t>(p) * D + j), acc[j]);
          }
          store_row<D, OUT_F32>(a, seq, qh, col, acc, Ls > 0.f ? 1.f / Ls : 0.f);
          if (lane == 0) a.arrive[unit] = 0;
        }
      }
    }
    fence_proxy_async_smem();  // this slot's reads are ordered before a bulk copy refills it
    __syncwarp();
    ++consumed;
    if (issue(slot)) ++issued;
  }
  if (timed_out) {
    if (lane == 0) set_status(a.status, PKV_DEV_TIMEOUT);
    // Let copies already in flight into this warp's ring land before the CTA exits.
    for (int n = consumed; n < issued; ++n) mbar_wait(&ring.full[n % STAGES], (n / STAGES) & 1);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

constexpr int kSimtWarps = PKV_SIMT_WARPS;
constexpr int kSimtStages = PKV_SIMT_STAGES;
constexpr int kSimtStages8 = PKV_SIMT_STAGES8;

template <int D, bool OUT_F32, bool KV8 = false>
static int launch_simt(const DecodeArgs& a, cudaStream_t stream) {
  constexpr int stages = KV8 ? kSimtStages8 : kSimtStages;
  auto kernel = decode_simt_kernel<D, OUT_F32, kSimtWarps, stages, KV8>;
  const size_t smem = sizeof(WarpRing<D, stages, KV8>) * kSimtWarps;
  static PerDevice<int> setup;  // blocks per SM, found once on each device
  int dev = 0, sms = 0, blocks_per_sm = 0;
  cudaError_t de = cudaGetDevice(&dev);
  if (de != cudaSuccess) return set_error(PKV_ERR_CUDA, "decode (simt): cudaGetDevice: %s", cudaGetErrorString(de));
  const int st = setup.get(
      dev,
      [&](int& bps) {
        cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (r == cudaSuccess) r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, kernel, kSimtWarps * 32, smem);
        return static_cast<int>(r);
      },
      &blocks_per_sm, static_cast<int>(cudaErrorInvalidDevice));
  if (st != 0)
    return set_error(PKV_ERR_CUDA, "decode (simt) setup: %s", cudaGetErrorString(static_cast<cudaError_t>(st)));
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::max(1, sms * std::max(1, blocks_per_sm));
  cudaError_t e = launch_after_previous(kernel, dim3(grid), dim3(kSimtWarps * 32), smem, stream, a);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "decode (simt) launch: %s", cudaGetErrorString(e));
  return PKV_OK;
}

int launch_decode_simt(const DecodeArgs& a, int head_dim, bool out_f32, cudaStream_t stream) {
  if (a.key_cache8) return out_f32 ? launch_simt<128, true, true>(a, stream) : launch_simt<128, false, true>(a, stream);
  if (head_dim == 128) return out_f32 ? launch_simt<128, true>(a, stream) : launch_simt<128, false>(a, stream);
  return out_f32 ? launch_simt<64, true>(a, stream) : launch_simt<64, false>(a, stream);
}

int launch_decode_plan(const DecodeArgs& a, const int32_t* context_lens, int max_context_len, cudaStream_t stream) {
  plan_kernel<<<1, kPlanThreads, 0, stream>>>(context_lens, a.num_seqs, max_context_len,
                                              a.max_blocks * a.block_size, a.partition,
                                              const_cast<PlanEntry*>(a.entries),
                                              const_cast<int32_t*>(a.plan_count), a.arrive,
                                              a.num_seqs * a.num_heads, a.status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "decode plan launch: %s", cudaGetErrorString(e));
  return PKV_OK;
}

static bool valid_partition(int p) {
  return p == 64 || p == 128 || p == 256 || p == 512 || p == 1024 || p == 2048;
}

// Split size for one call: the caller's choice if given (checked against the
// path's table-slice limit), else the path's automatic choice.  -1: invalid,
// -2: not supported by the chosen path.
static int resolve_partition(int partition_tokens, bool tensor, int num_seqs, int num_kv_heads, int block_size,
                             int max_context_len) {
  if (partition_tokens == 0)
    return tensor ? auto_partition_tokens_tensor(num_seqs, num_kv_heads, block_size, max_context_len)
                  : auto_partition_tokens(num_seqs, num_kv_heads, block_size, max_context_len);
  if (!valid_partition(partition_tokens) || partition_tokens % block_size != 0) return -1;
  if (!tensor && partition_tokens / block_size > 32) return -2;
  return partition_tokens;
}

}  // namespace pkv

using namespace pkv;

extern "C" int pkv_paged_attention_partition_tokens(int num_seqs, int num_kv_heads, int block_size,
                                                    int max_context_len) {
  if (num_seqs < 0 || num_kv_heads <= 0 || (block_size != 16 && block_size != 32) || max_context_len < 0)
    return set_error(PKV_ERR_INVALID, "partition_tokens: bad arguments");
  return auto_partition_tokens(num_seqs, num_kv_heads, block_size, max_context_len);
}

extern "C" size_t pkv_paged_attention_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                                     int block_size, int max_context_len, int partition_tokens) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
      (block_size != 16 && block_size != 32))
    return 0;
  // sized for the CUDA-core split, the shortest (so the largest workspace) of the two paths
  const int p = partition_tokens == 0 ? auto_partition_tokens(num_seqs, num_kv_heads, block_size, max_context_len)
                                      : resolve_partition(partition_tokens, true, num_seqs, num_kv_heads, block_size,
                                                          max_context_len);
  if (p < 0) return 0;
  return workspace_layout(num_seqs, num_heads, head_dim, max_context_len, p, false, num_kv_heads).total;
}

// Shared by the bf16 and the 8-bit entry points; `k_scale` != null selects the
// 8-bit (e4m3) pool (head_dim 128), read by the CUDA-core kernel or, for grouped
// query heads, by the tensor-core kernel that widens each tile to f16.
namespace pkv {
// The checks of a decode call that need no pointer: sizes, output type, path and partition.
// Returns PKV_OK (and the partition to use in *partition_out) or the call's error code.
int decode_check_sizes(int out_dtype, bool kv8, int max_blocks_per_seq, int max_context_len, int num_seqs,
                       int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                       int partition_tokens, int path, int* partition_out) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 ||
      max_context_len < 0)
    return set_error(PKV_ERR_INVALID, "paged_attention_decode: bad sizes");
  if (num_seqs > 65535 * 1024) return set_error(PKV_ERR_INVALID, "paged_attention_decode: too many sequences");
  if (out_dtype != PKV_DTYPE_BF16 && out_dtype != PKV_DTYPE_F32)
    return set_error(PKV_ERR_INVALID, "paged_attention_decode: out_dtype %d", out_dtype);
  if (head_dim != 64 && head_dim != 128)
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_decode: head_dim %d not in {64,128}", head_dim);
  if (block_size != 16 && block_size != 32)
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_decode: block_size %d not in {16,32}", block_size);
  if (num_kv_heads > 65535)  // the tensor-core kernels carry the kv head in 16 bits of their stage metadata
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_decode: num_kv_heads %d above 65535", num_kv_heads);
  if (num_heads % num_kv_heads != 0)
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_decode: num_heads %d not a multiple of num_kv_heads %d",
                     num_heads, num_kv_heads);
  if (path != PKV_PATH_AUTO && path != PKV_PATH_SIMT && path != PKV_PATH_TENSOR)
    return set_error(PKV_ERR_INVALID, "paged_attention_decode: path %d", path);
  if (kv8 && head_dim != 128)
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_decode_fp8: head_dim %d (only 128)", head_dim);
  const int group = num_heads / num_kv_heads;
  if (path == PKV_PATH_TENSOR && !tensor_path_supports(group, head_dim))
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_decode: tensor path needs 2 <= group <= 16 and head_dim 128"
                     " (group %d, head_dim %d)", group, head_dim);
  const bool use_tensor = path == PKV_PATH_TENSOR || (path == PKV_PATH_AUTO && tensor_path_supports(group, head_dim));
  const int partition =
      resolve_partition(partition_tokens, use_tensor, num_seqs, num_kv_heads, block_size, max_context_len);
  if (partition == -1)
    return set_error(PKV_ERR_INVALID, "paged_attention_decode: partition_tokens %d (64..2048, a power of two and a "
                     "multiple of block_size)", partition_tokens);
  if (partition == -2)
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_decode: the CUDA-core path splits at most 32 blocks "
                     "(partition_tokens %d, block_size %d)", partition_tokens, block_size);
  if (static_cast<int64_t>(max_context_len) > static_cast<int64_t>(65535) * partition)
    return set_error(PKV_ERR_INVALID, "paged_attention_decode: max_context_len too large for the split");
  *partition_out = partition;
  return PKV_OK;
}
}  // namespace pkv

static int decode_impl(void* out, int out_dtype, const void* query, const void* key_cache, const void* value_cache,
                       const float* k_scale, const float* v_scale, const int32_t* block_tables,
                       int max_blocks_per_seq, const int32_t* context_lens, int max_context_len, int num_seqs,
                       int num_heads, int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                       int partition_tokens, int path, void* workspace, size_t workspace_bytes, int32_t* status,
                       pkv_stream_t stream) {
  const bool kv8 = k_scale != nullptr;
  int partition = 0;
  const int rc_sizes = decode_check_sizes(out_dtype, kv8, max_blocks_per_seq, max_context_len, num_seqs, num_heads,
                                          num_kv_heads, head_dim, block_size, num_blocks, partition_tokens, path, &partition);
  if (rc_sizes != PKV_OK) return rc_sizes;
  const int group = num_heads / num_kv_heads;
  const bool use_tensor = path == PKV_PATH_TENSOR || (path == PKV_PATH_AUTO && tensor_path_supports(group, head_dim));
  if (num_seqs == 0) return PKV_OK;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens || !workspace ||
      (kv8 && !v_scale))
    return set_error(PKV_ERR_INVALID, "paged_attention_decode: null pointer");
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache))
    return set_error(PKV_ERR_INVALID, "paged_attention_decode: tensors must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return set_error(PKV_ERR_INVALID, "paged_attention_decode: workspace must be 256-byte aligned");
  const WorkspaceLayout w =
      workspace_layout(num_seqs, num_heads, head_dim, max_context_len, partition, false, num_kv_heads);
  if (workspace_bytes < w.total)
    return set_error(PKV_ERR_INVALID, "paged_attention_decode: workspace of %zu bytes, %zu needed", workspace_bytes,
                     w.total);
  if (static_cast<int64_t>(num_blocks) * num_kv_heads * block_size > (static_cast<int64_t>(1) << 31))
    return set_error(PKV_ERR_INVALID, "paged_attention_decode: pool too large");

  unsigned char* ws = static_cast<unsigned char*>(workspace);
  DecodeArgs a{};
  a.out = out;
  a.query = static_cast<const __nv_bfloat16*>(query);
  if (kv8) {
    a.key_cache8 = static_cast<const uint8_t*>(key_cache);
    a.value_cache8 = static_cast<const uint8_t*>(value_cache);
    a.k_scale = k_scale;
    a.v_scale = v_scale;
  } else {
    a.key_cache = static_cast<const __nv_bfloat16*>(key_cache);
    a.value_cache = static_cast<const __nv_bfloat16*>(value_cache);
  }
  a.block_tables = block_tables;
  a.plan_count = reinterpret_cast<const int32_t*>(ws + w.off_count);
  a.entries = reinterpret_cast<const PlanEntry*>(ws + w.off_entries);
  a.arrive = reinterpret_cast<int32_t*>(ws + w.off_arrive);
  a.part_o = reinterpret_cast<float*>(ws + w.off_part_o);
  a.part_ml = reinterpret_cast<float2*>(ws + w.off_part_ml);
  if (kv8 && use_tensor) {
    a.q_split = ws + w.off_qsplit;
    a.q_inv = reinterpret_cast<float*>(ws + w.off_qinv);
  }
  a.status = status;
  a.context_lens = context_lens;
  a.max_context_len = max_context_len;
  a.max_blocks = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.group = group;
  a.partition = partition;
  a.max_parts = w.max_parts;
  a.scale_log2 = scale * 1.4426950408889634f;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int rc = launch_decode_plan(a, context_lens, max_context_len, s);
  if (rc != PKV_OK) return rc;
  const bool out_f32 = out_dtype == PKV_DTYPE_F32;
  if (kv8 && use_tensor) return launch_decode_tensor_fp8(a, head_dim, out_f32, s);
  if (kv8) return out_f32 ? launch_simt<128, true, true>(a, s) : launch_simt<128, false, true>(a, s);
  if (use_tensor) return launch_decode_tensor(a, head_dim, out_f32, s);
  if (head_dim == 128) return out_f32 ? launch_simt<128, true>(a, s) : launch_simt<128, false>(a, s);
  return out_f32 ? launch_simt<64, true>(a, s) : launch_simt<64, false>(a, s);
}

extern "C" int pkv_paged_attention_decode(void* out, int out_dtype, const void* query, const void* key_cache,
                                          const void* value_cache, const int32_t* block_tables,
                                          int max_blocks_per_seq, const int32_t* context_lens,
                                          int max_context_len, int num_seqs, int num_heads, int num_kv_heads,
                                          int head_dim, int block_size, int num_blocks, float scale,
                                          int partition_tokens, int path, void* workspace, size_t workspace_bytes,
                                          int32_t* status, pkv_stream_t stream) {
  clear_error();
  return decode_impl(out, out_dtype, query, key_cache, value_cache, nullptr, nullptr, block_tables,
                     max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads, num_kv_heads, head_dim,
                     block_size, num_blocks, scale, partition_tokens, path, workspace, workspace_bytes, status,
                     stream);
}

extern "C" int pkv_paged_attention_decode_fp8(void* out, int out_dtype, const void* query, const void* key_cache,
                                              const void* value_cache, const float* k_scale, const float* v_scale,
                                              const int32_t* block_tables, int max_blocks_per_seq,
                                              const int32_t* context_lens, int max_context_len, int num_seqs,
                                              int num_heads, int num_kv_heads, int head_dim, int block_size,
                                              int num_blocks, float scale, int partition_tokens, int path,
                                              void* workspace, size_t workspace_bytes, int32_t* status,
                                              pkv_stream_t stream) {
  clear_error();
  if (!k_scale) return set_error(PKV_ERR_INVALID, "paged_attention_decode_fp8: null k_scale");
  return decode_impl(out, out_dtype, query, key_cache, value_cache, k_scale, v_scale, block_tables,
                     max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads, num_kv_heads, head_dim,
                     block_size, num_blocks, scale, partition_tokens, path, workspace, workspace_bytes,
                     status, stream);
}
