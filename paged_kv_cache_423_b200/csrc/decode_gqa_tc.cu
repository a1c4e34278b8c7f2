// Tensor-core (tcgen05) decode for grouped query heads.
//
// With g = num_heads / num_kv_heads > 1 every K and V row of a kv head serves g
// query heads: q·Kᵀ becomes a [tokens x g] product and P·V a [g x head_dim] one,
// dense contractions with g-wide operands.  This kernel runs both on the 5th-gen
// tensor cores with the accumulators in tensor memory, and keeps the online
// softmax (intelliparadigm article "PagedAttention：操作系统分页思想的跨界创新" §2.1:
// softmax(q·Kᵀ)·V over the pages of the block table) on the CUDA cores.
//
// Work item = (sequence, partition, kv head), handed out from the same sorted plan
// as the CUDA-core kernel.  A tile is 128 tokens = 8 slices of 16 rows; each slice
// of a (block, kv head) tile arrives by TMA (2-D tensor map over the pool viewed as
// [num_blocks * Hkv * block_size, head_dim], box 64 x 16, 128-byte swizzle), which
// is exactly the K-major operand layout of the MMA.  Per tile:
//   S[128 x N]  = K[128 x D] · Q[N x D]ᵀ          (A = K, K-major; B = Q, K-major)
//   softmax over the 128 rows of each of the g columns (fp32, base 2, online)
//   O[D x N]    = Vᵀ[D x 128] · P[128 x N]         (A = V, MN-major; B = P, K-major)
//   o_acc = o_acc * alpha + O                      (registers, thread = output row)
// N = 16 (the smallest MMA width for M = 128; g <= 16 query heads, the unused
// columns of Q are ignored and their P is 0).
// P is rounded to bf16 for the MMA; the softmax denominators sum the same rounded
// values, so the result is an exactly normalised attention with weights perturbed
// by at most 2^-9 relative.
//
// Roles: warps 0-3 (one thread per TMEM lane) do softmax and the output update and
// thread 0 issues the MMAs; warp 4 is the TMA producer, running up to STAGES tiles
// ahead across item boundaries.  Every wait is bounded; on a timeout the CTA stops,
// flags PKV_DEV_TIMEOUT, lets its copies land, frees its tensor memory and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "decode_common.cuh"
#include "pkv_internal.h"

namespace pkv {

namespace tc {

constexpr int kTile = 128;             // tokens per tile (MMA M)
constexpr int kChunk = 16;             // rows per TMA box
constexpr int kChunks = kTile / kChunk;
constexpr int kD = 128;                // head_dim of this path
constexpr int kHalfBytes = kTile * 128;  // one 64-column half of a K or V tile: 16 KiB
constexpr int kTileBytes = 2 * kHalfBytes;
constexpr int kConsumers = 128;        // warps 0-3
constexpr int kThreads = kConsumers + 32;
constexpr int kTmemCols = 32;          // S in columns [0,16), O in [16,32)
constexpr uint32_t kChunkTx = 4 * kChunk * 128;  // K and V, two halves each

struct alignas(64) Args {
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_q;
  DecodeArgs a;
};

// ---- PTX wrappers --------------------------------------------------------

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(smem_result)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] · B[smem desc], kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                     bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

// Arrive once on `bar` when every previously issued MMA of this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

template <int N>
__device__ __forceinline__ void tmem_load_row(uint32_t taddr, float (&v)[N]) {
  uint32_t r[N];
  if constexpr (N == 8) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
  } else {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  }
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < N; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void named_barrier_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Shared-memory matrix descriptor (sm_100 layout): start, leading/stride byte
// offsets (16-byte units), version 1, swizzle mode 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFF) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, A/B major-ness,
// N >> 3 and M >> 4.
__host__ __device__ constexpr uint32_t instr_desc(int m, int n, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn_major ? 1u << 15 : 0u) | (b_mn_major ? 1u << 16 : 0u) |
         (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// ---- shared memory layout -------------------------------------------------

template <int STAGES, int N>
struct Layout {
  static constexpr int kQBytes = 2 * N * 128;             // two 64-column halves, N rows each
  static constexpr int kQSlots = STAGES + 1;              // indexed by the CTA's item ordinal
  static constexpr int off_k = 0;
  static constexpr int off_v = off_k + STAGES * kTileBytes;
  static constexpr int off_q = off_v + STAGES * kTileBytes;
  static constexpr int off_p = off_q + kQSlots * 4096;    // q slots sized for N <= 16
  static constexpr int off_red = off_p + 4096;            // P: 2 K-atoms of N rows x 128 B
  static constexpr int off_meta = off_red + 2 * 4 * 16 * 4;
  static constexpr int off_bar = off_meta + STAGES * 16;
  static constexpr int off_misc = off_bar + (2 * STAGES + 2) * 8;
  static constexpr int bytes = off_misc + 16;
  static constexpr int alloc = bytes + 1024;              // slack to align the base to 1024
};

template <bool OUT_F32>
__device__ __forceinline__ void store_out(const DecodeArgs& a, int64_t idx, float v) {
  if constexpr (OUT_F32)
    static_cast<float*>(a.out)[idx] = v;
  else
    static_cast<__nv_bfloat16*>(a.out)[idx] = __float2bfloat16_rn(v);
}

// Column-wise maximum over the 32 rows a warp holds, for 16 columns at once: a
// transposed butterfly (16 shuffles) that leaves column (lane >> 1) in both lanes
// of each pair.
__device__ __forceinline__ float warp_colmax16(const float (&x)[16], int lane) {
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool up = lane & 16;
    const float send = up ? x[i] : x[i + 8];
    const float keep = up ? x[i + 8] : x[i];
    v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 16));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool up = lane & 8;
    const float send = up ? v[i] : v[i + 4];
    const float keep = up ? v[i + 4] : v[i];
    v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 8));
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool up = lane & 4;
    const float send = up ? v[i] : v[i + 2];
    const float keep = up ? v[i + 2] : v[i];
    v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 4));
  }
  {
    const bool up = lane & 2;
    const float send = up ? v[0] : v[1];
    const float keep = up ? v[1] : v[0];
    v[0] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 2));
  }
  return fmaxf(v[0], __shfl_xor_sync(0xffffffffu, v[0], 1));
}

// meta.w bits: n_valid (8) | chunk mask << 8 (8) | first << 16 | last << 17 | with_q << 18
template <int STAGES, int N, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1) decode_gqa_tc_kernel(const __grid_constant__ Args args) {
  static_assert(N == 16, "the tile is M = 128 rows, whose narrowest MMA is N = 16");
  using L = Layout<STAGES, N>;
  const DecodeArgs& a = args.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* k_ring = smem + L::off_k;
  unsigned char* v_ring = smem + L::off_v;
  unsigned char* q_ring = smem + L::off_q;
  unsigned char* p_tile = smem + L::off_p;
  float* red = reinterpret_cast<float*>(smem + L::off_red);  // [2][4 warps][16]
  int4* meta = reinterpret_cast<int4*>(smem + L::off_meta);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  uint64_t* empty = full + STAGES;
  uint64_t* s_bar = empty + STAGES;   // S of a tile is ready
  uint64_t* o_bar = s_bar + 1;        // O of a tile is ready
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::off_misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::off_misc + 4);
  int* merge_flag = reinterpret_cast<int*>(smem + L::off_misc + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = a.group;
  const int64_t n_items = static_cast<int64_t>(a.plan_count[0]) * a.num_kv_heads;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(s_bar, 1);
    mbar_init(o_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // P rows of unused heads (g..N-1) stay zero for the whole kernel.
  for (int i = tid; i < 4096 / 16; i += blockDim.x) reinterpret_cast<uint4*>(p_tile)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ================= producer =================
    const uint64_t policy = l2_policy_evict_first();
    int n = 0;  // fills issued
    int item_ord = 0;
    for (int64_t item = blockIdx.x; item < n_items && !*abort_flag; item += gridDim.x, ++item_ord) {
      const PlanEntry e = a.entries[item / a.num_kv_heads];
      const int kvh = static_cast<int>(item % a.num_kv_heads);
      const int tok0 = e.y * a.partition;
      const int ntok = e.w == 0 ? 0 : min(a.partition, e.w - tok0);
      const int nblk = (ntok + a.block_size - 1) / a.block_size;
      const int tab = lane < nblk ? __ldg(a.block_tables + static_cast<int64_t>(e.x) * a.max_blocks + tok0 / a.block_size + lane) : 0;
      const int ntiles = ntok == 0 ? 1 : (ntok + kTile - 1) / kTile;
      for (int tile = 0; tile < ntiles; ++tile, ++n) {
        const int slot = n % STAGES;
        if (n >= STAGES && !mbar_wait(&empty[slot], ((n / STAGES) - 1) & 1)) {
          *abort_flag = 1;
          set_status(a.status, PKV_DEV_TIMEOUT);
          break;
        }
        const int n_valid = max(0, min(kTile, ntok - tile * kTile));
        const int nchunks = (n_valid + kChunk - 1) / kChunk;
        const int ltok = tile * kTile + lane * kChunk;  // this lane's chunk (lane < nchunks)
        const int phys = __shfl_sync(0xffffffffu, tab, min(31, ltok / a.block_size));
        const bool mine = lane < nchunks;
        const bool ok = mine && phys >= 0 && phys < a.num_blocks;
        const uint32_t mask = __ballot_sync(0xffffffffu, ok);
        if (mine && !ok) set_status(a.status, PKV_DEV_BAD_BLOCK);
        const bool with_q = tile == 0 && ntok > 0;
        if (lane == 0) {
          meta[slot] = make_int4(e.x, kvh, e.y | (e.z << 16),
                                 n_valid | (mask << 8) | (tile == 0 ? 1 << 16 : 0) | (tile == ntiles - 1 ? 1 << 17 : 0) |
                                     (with_q ? 1 << 18 : 0));
          mbar_arrive_expect_tx(&full[slot], __popc(mask) * kChunkTx + (with_q ? L::kQBytes : 0));
        }
        __syncwarp();
        if (ok) {
          const int row = (phys * a.num_kv_heads + kvh) * a.block_size + ltok % a.block_size;
          unsigned char* kd = k_ring + slot * kTileBytes + lane * kChunk * 128;
          unsigned char* vd = v_ring + slot * kTileBytes + lane * kChunk * 128;
          tma_load_2d(kd, &args.tm_k, 0, row, &full[slot], policy);
          tma_load_2d(kd + kHalfBytes, &args.tm_k, 64, row, &full[slot], policy);
          tma_load_2d(vd, &args.tm_v, 0, row, &full[slot], policy);
          tma_load_2d(vd + kHalfBytes, &args.tm_v, 64, row, &full[slot], policy);
        }
        if (with_q && lane == 0) {
          // The producer runs at most STAGES tiles (so STAGES items) ahead of the
          // consumers: STAGES + 1 q slots never overwrite the q still in use.
          const int qrow = e.x * a.num_heads + kvh * g;
          unsigned char* qd = q_ring + (item_ord % L::kQSlots) * 4096;
          tma_load_2d(qd, &args.tm_q, 0, qrow, &full[slot], policy);
          tma_load_2d(qd + N * 128, &args.tm_q, 64, qrow, &full[slot], policy);
        }
      }
    }
    // Let this CTA's last copies land before the final barrier.
    for (int k = max(0, n - STAGES); k < n; ++k) mbar_wait(&full[k % STAGES], (k / STAGES) & 1);
  } else {
    // ================= consumers (one thread per TMEM lane) =================
    constexpr uint32_t idesc_qk = instr_desc(kTile, N, false, false);
    constexpr uint32_t idesc_pv = instr_desc(kD, N, true, false);
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tmem_s = tmem + lane_base;
    const uint32_t tmem_o = tmem + lane_base + 16;
    const uint32_t p_addr = smem_addr(p_tile);

    // S = K · Qᵀ for the tile in `slot` (thread 0 only).
    auto issue_qk = [&](int slot, int ord) {
      const uint32_t k_addr = smem_addr(k_ring + slot * kTileBytes);
      const uint32_t q_addr = smem_addr(q_ring + (ord % L::kQSlots) * 4096);
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t koff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
        const uint32_t qoff = (kk >> 2) * (N * 128) + (kk & 3) * 32;
        umma(tmem, smem_desc_sw128(k_addr + koff, 16, 1024), smem_desc_sw128(q_addr + qoff, 16, 1024), idesc_qk,
             kk > 0);
      }
      umma_commit(s_bar);
    };

    float m[N], lp[N], oacc[N], alpha[N];
#pragma unroll
    for (int h = 0; h < N; ++h) m[h] = -INFINITY, lp[h] = 0.f, oacc[h] = 0.f, alpha[h] = 1.f;
    int s_phase = 0, o_phase = 0;
    int n = 0;
    int item_ord = 0;
    // Thread 0 issues the first tile's S before the loop; afterwards S of tile n+1
    // is issued right behind O of tile n, so the tensor core computes it while the
    // other threads finish tile n.
    if (tid == 0 && n_items > blockIdx.x) {
      if (!mbar_wait(&full[0], 0)) *abort_flag = 1;
      else if ((meta[0].w & 0xff) > 0) issue_qk(0, 0);
    }
    for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x, ++item_ord) {
      const PlanEntry e = a.entries[item / a.num_kv_heads];
      const int ntok = e.w == 0 ? 0 : min(a.partition, e.w - e.y * a.partition);
      const int ntiles = ntok == 0 ? 1 : (ntok + kTile - 1) / kTile;
      const bool more_items = item + gridDim.x < n_items;
      bool stop = false;
      for (int tile = 0; tile < ntiles; ++tile, ++n) {
        const int slot = n % STAGES;
        if (!mbar_wait(&full[slot], (n / STAGES) & 1)) *abort_flag = 1;
        named_barrier_sync(1, kConsumers);
        if (*abort_flag) {
          stop = true;
          break;
        }
        const int4 mt = meta[slot];
        const int n_valid = mt.w & 0xff;
        const uint32_t mask = (mt.w >> 8) & 0xff;
        const bool first = (mt.w >> 16) & 1, last = (mt.w >> 17) & 1;
        if (first) {
#pragma unroll
          for (int h = 0; h < N; ++h) m[h] = -INFINITY, lp[h] = 0.f, oacc[h] = 0.f;
        }
        // the tile after this one (in this CTA's stream), whose S thread 0 issues early
        const bool has_next = tile + 1 < ntiles || more_items;
        const int next_slot = (n + 1) % STAGES;
        const int next_ord = tile + 1 < ntiles ? item_ord : item_ord + 1;
        if (n_valid > 0) {
          const uint32_t v_addr = smem_addr(v_ring + slot * kTileBytes);
          if (!mbar_wait(s_bar, s_phase)) *abort_flag = 1;
          s_phase ^= 1;
          tc_fence_after();
          float s[N];
          tmem_load_row<N>(tmem_s, s);
          // ---- online softmax over this tile's rows, per query head (column)
          const int t = tid;  // this thread's row = token of the tile
          const bool valid = t < n_valid && ((mask >> (t / kChunk)) & 1);
          float x[N];
#pragma unroll
          for (int h = 0; h < N; ++h) x[h] = (valid && h < g) ? s[h] * a.scale_log2 : -INFINITY;
          const float wmax = warp_colmax16(x, lane);
          if ((lane & 1) == 0) red[warp * 16 + (lane >> 1)] = wmax;
          named_barrier_sync(1, kConsumers);
#pragma unroll
          for (int h = 0; h < N; ++h) {
            if (h >= g) break;
            const float tmax = fmaxf(fmaxf(red[h], red[16 + h]), fmaxf(red[32 + h], red[48 + h]));
            const float m_new = fmaxf(m[h], tmax);
            alpha[h] = m_new == -INFINITY ? 1.f : exp2f(m[h] - m_new);
            m[h] = m_new;
            const float p = valid ? exp2f(x[h] - m_new) : 0.f;
            const __nv_bfloat16 pb = __float2bfloat16_rn(p);
            lp[h] = fmaf(lp[h], alpha[h], __bfloat162float(pb));
            // P[t][h] into the K-major, 128-byte-swizzled B operand (rows = heads)
            const int katom = t >> 6, chunk = (t & 63) >> 3;
            const int off = katom * (N * 128) + h * 128 + ((chunk ^ (h & 7)) << 4) + ((t & 7) << 1);
            *reinterpret_cast<__nv_bfloat16*>(p_tile + off) = pb;
          }
          if (!valid) {
            // rows of V outside the context may hold anything (even NaN): zero them
            uint4* r0 = reinterpret_cast<uint4*>(v_ring + slot * kTileBytes + t * 128);
            uint4* r1 = reinterpret_cast<uint4*>(v_ring + slot * kTileBytes + kHalfBytes + t * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) r0[c] = r1[c] = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          named_barrier_sync(1, kConsumers);
          if (tid == 0) {
            // ---- O = Vᵀ · P over the tile's valid 16-row slices
            tc_fence_after();
            const int kt = (n_valid + 15) / 16;
            for (int kk = 0; kk < kt; ++kk) {
              const uint32_t poff = (kk >> 2) * (N * 128) + (kk & 3) * 32;
              umma(tmem + 16, smem_desc_sw128(v_addr + kk * 2048, kHalfBytes, 1024),
                   smem_desc_sw128(p_addr + poff, 16, 1024), idesc_pv, kk > 0);
            }
            umma_commit(o_bar);
            umma_commit(&empty[slot]);
            // ---- S of the next tile (S of this tile has been read by every thread)
            if (has_next) {
              if (!mbar_wait(&full[next_slot], ((n + 1) / STAGES) & 1)) *abort_flag = 1;
              else if ((meta[next_slot].w & 0xff) > 0) issue_qk(next_slot, next_ord);
            }
          }
          if (!mbar_wait(o_bar, o_phase)) *abort_flag = 1;
          o_phase ^= 1;
          tc_fence_after();
          float o[N];
          tmem_load_row<N>(tmem_o, o);
#pragma unroll
          for (int h = 0; h < N; ++h) oacc[h] = fmaf(oacc[h], alpha[h], o[h]);
          tc_fence_before();
        } else if (tid == 0) {
          mbar_arrive(&empty[slot]);  // nothing to compute: hand the stage back
          if (has_next) {
            if (!mbar_wait(&full[next_slot], ((n + 1) / STAGES) & 1)) *abort_flag = 1;
            else if ((meta[next_slot].w & 0xff) > 0) issue_qk(next_slot, next_ord);
          }
        }
        if (last) {
          // ---- finalize the item: softmax denominators, then the output (or a partial)
          float* red2 = red + 64;
#pragma unroll
          for (int h = 0; h < N; ++h) {
            if (h >= g) break;
            float w = lp[h];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) w += __shfl_xor_sync(0xffffffffu, w, off);
            if (lane == 0) red2[warp * 16 + h] = w;
          }
          named_barrier_sync(1, kConsumers);
          const int seq = mt.x, kvh = mt.y, part = mt.z & 0xffff, nparts = mt.z >> 16;
          const int d = tid;
          if (nparts == 1) {
#pragma unroll
            for (int h = 0; h < N; ++h) {
              if (h >= g) break;
              const float l = red2[h] + red2[16 + h] + red2[32 + h] + red2[48 + h];
              store_out<OUT_F32>(a, (static_cast<int64_t>(seq) * a.num_heads + kvh * g + h) * kD + d,
                                 l > 0.f ? oacc[h] / l : 0.f);
            }
          } else {
            const int64_t unit0 = static_cast<int64_t>(seq) * a.num_heads + kvh * g;
#pragma unroll
            for (int h = 0; h < N; ++h) {
              if (h >= g) break;
              const float l = red2[h] + red2[16 + h] + red2[32 + h] + red2[48 + h];
              const int64_t pidx = (unit0 + h) * a.max_parts + part;
              a.part_o[pidx * kD + d] = oacc[h];
              if (d == 0) a.part_ml[pidx] = make_float2(m[h], l);
            }
            __threadfence();
            named_barrier_sync(1, kConsumers);
            if (tid == 0) *merge_flag = atomicAdd(a.arrive + unit0, 1) == nparts - 1;
            named_barrier_sync(1, kConsumers);
            if (*merge_flag) {
              __threadfence();
              for (int h = 0; h < g; ++h) {
                const float2* ml = a.part_ml + (unit0 + h) * a.max_parts;
                const float* po = a.part_o + (unit0 + h) * a.max_parts * kD + d;
                float M = -INFINITY;
                for (int p = 0; p < nparts; ++p) M = fmaxf(M, __ldcg(&ml[p].x));
                float acc = 0.f, Ls = 0.f;
                for (int p = 0; p < nparts; ++p) {
                  const float2 mlp = __ldcg(&ml[p]);
                  const float w = exp2f(mlp.x - M);
                  Ls = fmaf(w, mlp.y, Ls);
                  acc = fmaf(w, __ldcg(po + static_cast<int64_t>(p) * kD), acc);
                }
                store_out<OUT_F32>(a, (unit0 + h) * kD + d, Ls > 0.f ? acc / Ls : 0.f);
              }
              if (tid == 0) a.arrive[unit0] = 0;
            }
          }
        }
      }
      if (stop) break;
    }
    if (*abort_flag && tid == 0) set_status(a.status, PKV_DEV_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---- host side -----------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D view [rows, 128] of a bf16 tensor, box 64 x box_rows, 128-byte swizzle.
static int encode_map(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows, const char* what) {
  auto encode = tensor_map_encoder();
  if (!encode) return set_error(PKV_ERR_CUDA, "decode (tensor): cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), rows};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(PKV_ERR_CUDA, "decode (tensor): tensor map for %s failed (%d)", what, (int)r);
  return PKV_OK;
}

constexpr int kStages = 3;

template <int N, bool OUT_F32>
static int launch(const Args& args, cudaStream_t stream) {
  auto kernel = decode_gqa_tc_kernel<kStages, N, OUT_F32>;
  const int smem = Layout<kStages, N>::alloc;
  static std::once_flag once;
  static cudaError_t setup = cudaSuccess;
  std::call_once(once, [&] { setup = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); });
  if (setup != cudaSuccess) return set_error(PKV_ERR_CUDA, "decode (tensor) setup: %s", cudaGetErrorString(setup));
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  kernel<<<std::max(1, sms), kThreads, smem, stream>>>(args);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "decode (tensor) launch: %s", cudaGetErrorString(e));
  return PKV_OK;
}

}  // namespace tc

bool tensor_path_supports(int group, int head_dim) { return head_dim == tc::kD && group >= 2 && group <= 16; }

int launch_decode_tensor(const DecodeArgs& a, int head_dim, bool out_f32, cudaStream_t stream) {
  if (!tensor_path_supports(a.group, head_dim))
    return set_error(PKV_ERR_UNSUPPORTED, "decode (tensor): group %d / head_dim %d not supported", a.group, head_dim);
  tc::Args args;
  args.a = a;
  constexpr int n = 16;
  const uint64_t pool_rows = static_cast<uint64_t>(a.num_blocks) * a.num_kv_heads * a.block_size;
  int rc = tc::encode_map(&args.tm_k, a.key_cache, pool_rows, tc::kChunk, "key_cache");
  if (rc == PKV_OK) rc = tc::encode_map(&args.tm_v, a.value_cache, pool_rows, tc::kChunk, "value_cache");
  if (rc == PKV_OK)
    rc = tc::encode_map(&args.tm_q, a.query, static_cast<uint64_t>(a.num_seqs) * a.num_heads, n, "query");
  if (rc != PKV_OK) return rc;
  return out_f32 ? tc::launch<n, true>(args, stream) : tc::launch<n, false>(args, stream);
}

}  // namespace pkv
