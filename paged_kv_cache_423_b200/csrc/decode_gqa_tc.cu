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
// as the CUDA-core kernel.  A tile is 128 tokens = 8 slices of 16 rows (4 of 32 when
// the block size is a multiple of 32); each slice of a (block, kv head) tile arrives
// by TMA (2-D tensor map over the pool viewed as [num_blocks * Hkv * block_size,
// head_dim], box 64 columns x 16 or 32 rows, 128-byte swizzle), which is exactly the
// K-major operand layout of the MMA.  The TMA engine's time per box is what limits a
// single producer warp, so the larger box is used wherever the pool allows it.  Per tile:
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

#include "decode_common.cuh"
#include "launch_setup.cuh"
#include "pkv_internal.h"
#include "tcgen05_common.cuh"

namespace pkv {

namespace tc {

constexpr int kTile = 128;             // tokens per tile (MMA M)
constexpr int kChunk = 16;             // rows per validity bit (and per TMA box at block size 16)
constexpr int kD = 128;                // head_dim of this path
constexpr int kHalfBytes = kTile * 128;  // one 64-column half of a K or V tile: 16 KiB
constexpr int kTileBytes = 2 * kHalfBytes;
constexpr int kConsumers = 128;        // warps 0-3: softmax, one thread per TMEM lane
constexpr int kProducerWarp = 4;       // TMA loads
constexpr int kMmaWarp = 5;            // tcgen05.mma issue
constexpr int kThreads = kConsumers + 64;
constexpr int kTmemCols = 64;          // S double buffer in columns [0,16) and [16,32), O of even / odd
constexpr uint32_t kColO = 32;         // items in [32,48) and [48,64)

struct alignas(64) Args {
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_q;
  DecodeArgs a;
};

// Rows per TMA box: 32 where every 32-row slice stays inside one block, else 16.
__host__ __device__ constexpr int box_rows(int block_size) { return block_size % 32 == 0 ? 32 : kChunk; }

// ---- shared memory layout -------------------------------------------------

template <int STAGES, int N>
struct Layout {
  static constexpr int kQBytes = 2 * N * 128;             // two 64-column halves, N rows each
  static constexpr int kQSlots = STAGES + 1;              // indexed by the CTA's item ordinal
  static constexpr int off_k = 0;
  static constexpr int off_v = off_k + STAGES * kTileBytes;
  static constexpr int off_q = off_v + STAGES * kTileBytes;
  static constexpr int off_p = off_q + kQSlots * 4096;    // q slots sized for N <= 16
  static constexpr int off_red = off_p + 2 * 4096;        // P double buffer: 2 K-atoms of N rows x 128 B each
  static constexpr int off_meta = off_red + 3 * 4 * 16 * 4;  // [maxima | sums of even items | odd items][4 warps][16]
  static constexpr int off_bar = off_meta + STAGES * 16;
  // full, empty, s_full[2], s_free[2], p_full[2], o_bar[2], drain
  static constexpr int kBars = 2 * STAGES + 9;
  static constexpr int off_misc = off_bar + kBars * 8;
  static constexpr int bytes = off_misc + 32;
  static constexpr int alloc = bytes + 1024;              // slack to align the base to 1024
};

template <bool OUT_F32>
__device__ __forceinline__ void store_out(const DecodeArgs& a, int64_t idx, float v) {
  if constexpr (OUT_F32)
    static_cast<float*>(a.out)[idx] = v;
  else
    static_cast<__nv_bfloat16*>(a.out)[idx] = __float2bfloat16_rn(v);
}

// Softmax rows are rescaled only when a score exceeds the held maximum by more
// than 2^kRescaleLog2 (weights up to 256 before normalisation, harmless in bf16
// and fp32); otherwise P uses the held maximum and P·V keeps accumulating in TMEM.
constexpr float kRescaleLog2 = 8.f;

// Stage metadata, written by the producer:
//   x = sequence, y = kv head | q slot << 16, z = partition | partitions << 16,
//   w = valid rows (8 bits) | chunk mask << 8 | first << 16 | last << 17 | end of stream << 18
constexpr int kMetaFirst = 1 << 16, kMetaLast = 1 << 17, kMetaEnd = 1 << 18;

// Pipeline (per CTA, persistent over work items):
//   producer warp  -> full[s]      : K, V (and q on an item's first tile) landed in stage s
//   MMA warp       -> s_full[b]    : S = K·Qᵀ of a tile is in TMEM buffer b (two buffers)
//   softmax warps  -> s_free[b]    : S buffer b has been read
//   softmax warps  -> p_full[b]    : P of the tile is in shared buffer b (two buffers)
//   MMA warp       -> o_bar[b]     : O += Vᵀ·P of that tile is done (P buffer b reusable)
//   MMA warp and the 4 softmax warps -> empty[s] : stage s may be refilled (its
//                    P·V is done and its metadata has been read; a tile with no
//                    valid rows must not be refilled before the softmax has seen it)
// The MMA warp never blocks on one side while the other could proceed: it polls
// both (QK of the next landed tile, PV of the next tile whose P is ready).
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
  unsigned char* p_buf = smem + L::off_p;                    // [2][4096]
  float* red = reinterpret_cast<float*>(smem + L::off_red);  // [2][4 warps][16]
  int4* meta = reinterpret_cast<int4*>(smem + L::off_meta);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::off_bar);
  uint64_t* empty = full + STAGES;
  uint64_t* s_full = empty + STAGES;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_bar = p_full + 2;
  uint64_t* drain = o_bar + 2;  // the MMA thread's last commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::off_misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::off_misc + 4);
  // [P buffer]: bit 0 = the P·V starts a fresh accumulation, bit 1 = the O buffer of its item
  volatile int* restart_flag = reinterpret_cast<volatile int*>(smem + L::off_misc + 8);  // [2]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = a.group;
  griddep_launch_dependents();  // the merge kernel may be scheduled now; it waits for this one to end

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 5);  // the MMA commit after P·V, and each softmax warp once it has read the metadata
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 4);  // one arrival per softmax warp
      mbar_init(&p_full[b], 4);
      mbar_init(&o_bar[b], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // P rows of unused heads (g..N-1) stay zero for the whole kernel.
  for (int i = tid; i < 2 * 4096 / 16; i += blockDim.x) reinterpret_cast<uint4*>(p_buf)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The set-up above overlaps the plan kernel; its work list is read only after it has finished.
  griddep_wait();
  const int64_t n_items = static_cast<int64_t>(a.plan_count[0]) * a.num_kv_heads;

  if (warp == kProducerWarp) {
    // ================= producer =================
    const uint64_t policy = l2_policy_kv();
    auto load_entry = [&](int64_t it) -> PlanEntry {
      return it < n_items ? a.entries[it / a.num_kv_heads] : make_int4(0, 0, 0, 0);
    };
    // The item's block-table slice: lane l holds entries l, l+32, l+64, l+96 (an
    // item spans at most 2048 tokens = 128 blocks of 16).
    auto load_tab = [&](const PlanEntry& e) -> int4 {
      const int tok0 = e.y * a.partition;
      const int ntok = e.w == 0 ? 0 : min(a.partition, e.w - tok0);
      const int nblk = (ntok + a.block_size - 1) / a.block_size;
      const int32_t* row = a.block_tables + static_cast<int64_t>(e.x) * a.max_blocks + tok0 / a.block_size +
                           (a.block_offset ? a.block_offset[e.x] : 0);
      int4 t = make_int4(0, 0, 0, 0);
      if (lane < nblk) t.x = __ldg(row + lane);
      if (lane + 32 < nblk) t.y = __ldg(row + lane + 32);
      if (lane + 64 < nblk) t.z = __ldg(row + lane + 64);
      if (lane + 96 < nblk) t.w = __ldg(row + lane + 96);
      return t;
    };
    // Items are taken from a global counter in plan order (longest first), so CTAs
    // that finish early take more.  The next item is claimed when the current one's last
    // tile is issued (its counter, entry and table slice then load while the ring
    // drains), not earlier: a claimed item waits for this CTA alone, so claiming ahead
    // would hold work back from CTAs that run out at the end.
    int* work_counter = const_cast<int*>(a.plan_count) + 1;
    auto grab = [&]() -> int64_t {
      int v = 0;
      if (lane == 0) v = atomicAdd(work_counter, 1);
      return __shfl_sync(0xffffffffu, v, 0);
    };
    int64_t item = grab();
    int64_t item_nxt = n_items;
    PlanEntry e_cur = load_entry(item);
    int4 tab_cur = item < n_items ? load_tab(e_cur) : make_int4(0, 0, 0, 0);
    const int crow = box_rows(a.block_size);
    int n = 0;  // fills issued
    int item_ord = 0;
    bool failed = false;
    auto acquire = [&](int slot) -> bool {
      if (n >= STAGES && !mbar_wait(&empty[slot], ((n / STAGES) - 1) & 1)) {
        *abort_flag = 1;
        set_status(a.status, PKV_DEV_TIMEOUT);
        return false;
      }
      return true;
    };
    while (item < n_items && !failed && !*abort_flag) {
      const PlanEntry e = e_cur;
      const int kvh = static_cast<int>(item % a.num_kv_heads);
      const int ntok = e.w == 0 ? 0 : min(a.partition, e.w - e.y * a.partition);
      const int ntiles = ntok == 0 ? 1 : (ntok + kTile - 1) / kTile;
      const int qslot = item_ord % L::kQSlots;
      for (int tile = 0; tile < ntiles; ++tile, ++n) {
        const int slot = n % STAGES;
        if (tile == ntiles - 1) item_nxt = grab();
        if (!acquire(slot)) {
          failed = true;
          break;
        }
        const int n_valid = max(0, min(kTile, ntok - tile * kTile));
        const int nchunks = (n_valid + crow - 1) / crow;
        const int ltok = tile * kTile + lane * crow;  // this lane's box (lane < nchunks)
        const int blk = min(127, ltok / a.block_size);
        const int p0 = __shfl_sync(0xffffffffu, tab_cur.x, blk & 31);
        const int p1 = __shfl_sync(0xffffffffu, tab_cur.y, blk & 31);
        const int p2 = __shfl_sync(0xffffffffu, tab_cur.z, blk & 31);
        const int p3 = __shfl_sync(0xffffffffu, tab_cur.w, blk & 31);
        const int phys = blk < 32 ? p0 : blk < 64 ? p1 : blk < 96 ? p2 : p3;
        const bool mine = lane < nchunks;
        const bool ok = mine && phys >= 0 && phys < a.num_blocks;
        const uint32_t boxes = __ballot_sync(0xffffffffu, ok);
        // validity per 16-row slice (a 32-row box covers two)
        uint32_t mask = boxes;
        if (crow == 32) {
          mask = 0;
#pragma unroll
          for (int i = 0; i < kTile / 32; ++i)
            if ((boxes >> i) & 1) mask |= 3u << (2 * i);
        }
        if (mine && !ok) set_status(a.status, PKV_DEV_BAD_BLOCK);
        const bool with_q = tile == 0 && ntok > 0;
        if (lane == 0) {
          meta[slot] = make_int4(e.x, kvh | (qslot << 16), e.y | (e.z << 16),
                                 n_valid | (mask << 8) | (tile == 0 ? kMetaFirst : 0) | (tile == ntiles - 1 ? kMetaLast : 0));
          // K and V of each landed box, two 64-column halves each
          mbar_arrive_expect_tx(&full[slot], __popc(boxes) * (4u * crow * 128u) + (with_q ? L::kQBytes : 0));
        }
        __syncwarp();
        if (ok) {
          const int row = (phys * a.num_kv_heads + kvh) * a.block_size + ltok % a.block_size;
          unsigned char* kd = k_ring + slot * kTileBytes + lane * crow * 128;
          unsigned char* vd = v_ring + slot * kTileBytes + lane * crow * 128;
          tma_load_2d(kd, &args.tm_k, 0, row, &full[slot], policy);
          tma_load_2d(kd + kHalfBytes, &args.tm_k, 64, row, &full[slot], policy);
          tma_load_2d(vd, &args.tm_v, 0, row, &full[slot], policy);
          tma_load_2d(vd + kHalfBytes, &args.tm_v, 64, row, &full[slot], policy);
        }
        if (with_q && lane == 0) {
          // The producer runs at most STAGES fills (so STAGES items) ahead of the
          // last released stage: STAGES + 1 q slots never overwrite a q in use.
          const int qrow = e.x * a.num_heads + kvh * g;
          unsigned char* qd = q_ring + qslot * 4096;
          tma_load_2d(qd, &args.tm_q, 0, qrow, &full[slot], policy);
          tma_load_2d(qd + N * 128, &args.tm_q, 64, qrow, &full[slot], policy);
        }
      }
      item = item_nxt;
      ++item_ord;
      e_cur = load_entry(item);
      tab_cur = item < n_items ? load_tab(e_cur) : make_int4(0, 0, 0, 0);
    }
    if (!failed && !*abort_flag) {
      // end-of-stream marker: a fill with no data
      const int slot = n % STAGES;
      if (acquire(slot)) {
        if (lane == 0) {
          meta[slot] = make_int4(0, 0, 0, kMetaEnd);
          mbar_arrive_expect_tx(&full[slot], 0);
        }
        ++n;
      }
      __syncwarp();
    }
    // Let this CTA's last copies land before the final barrier.
    for (int k = max(0, n - STAGES); k < n; ++k) mbar_wait(&full[k % STAGES], (k / STAGES) & 1);
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer (one thread) =================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = instr_desc(kTile, N, false, false);
      constexpr uint32_t idesc_pv = instr_desc(kD, N, true, true);
      const uint32_t p_addr0 = smem_addr(p_buf);
      int qk_n = 0, pv_n = 0, end_n = 0x7fffffff;
      int q_valid = 0, p_valid = 0;  // valid (non-empty) tiles that got their QK / PV
      uint64_t idle_since = 0;
      int idle = 0;
      while (pv_n < end_n) {
        bool progress = false;
        // ---- QK of the next landed tile, if its S buffer is free
        if (qk_n < end_n && mbar_test(&full[qk_n % STAGES], (qk_n / STAGES) & 1)) {
          const int4 mt = meta[qk_n % STAGES];
          if (mt.w & kMetaEnd) {
            end_n = qk_n;
            progress = true;
          } else if ((mt.w & 0xff) == 0) {
            ++qk_n;
            progress = true;
          } else {
            const int b = q_valid & 1;
            if (q_valid < 2 || mbar_test(&s_free[b], ((q_valid >> 1) - 1) & 1)) {
              tc_fence_after();
              const int slot = qk_n % STAGES;
              const uint32_t k_addr = smem_addr(k_ring + slot * kTileBytes);
              const uint32_t q_addr = smem_addr(q_ring + (mt.y >> 16) * 4096);
#pragma unroll
              for (int kk = 0; kk < kD / 16; ++kk) {
                const uint32_t koff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                const uint32_t qoff = (kk >> 2) * (N * 128) + (kk & 3) * 32;
                umma(tmem + b * 16, smem_desc_sw128(k_addr + koff, 16, 1024),
                     smem_desc_sw128(q_addr + qoff, 16, 1024), idesc_qk, kk > 0);
              }
              umma_commit(&s_full[b]);
              ++q_valid;
              ++qk_n;
              progress = true;
            }
          }
        }
        // ---- PV of the oldest tile whose P is ready
        if (pv_n < qk_n) {
          const int slot = pv_n % STAGES;
          const int4 mt = meta[slot];
          if ((mt.w & 0xff) == 0) {
            mbar_arrive(&empty[slot]);
            ++pv_n;
            progress = true;
          } else {
            const int b = p_valid & 1;
            if (mbar_test(&p_full[b], (p_valid >> 1) & 1)) {
              tc_fence_after();
              const int rf = restart_flag[b];
              const bool restart = rf & 1;
              const uint32_t o_col = kColO + ((rf >> 1) & 1) * 16;
              const uint32_t v_addr = smem_addr(v_ring + slot * kTileBytes);
              const uint32_t p_addr = p_addr0 + b * 4096;
              const int kt = ((mt.w & 0xff) + 15) / 16;
              for (int kk = 0; kk < kt; ++kk) {
                // P: MN-major, unswizzled; 8-token groups 128 B apart, heads 8..15 2 KiB on
                umma(tmem + o_col, smem_desc_sw128(v_addr + kk * 2048, kHalfBytes, 1024),
                     smem_desc_plain(p_addr + kk * 256, 128, 2048), idesc_pv, kk > 0 || !restart);
              }
              umma_commit(&o_bar[b]);
              umma_commit(&empty[slot]);
              ++p_valid;
              ++pv_n;
              progress = true;
            }
          }
        }
        if (progress) {
          idle = 0;
        } else {
          // Back off briefly: this warp shares its scheduler with a softmax warp.
          __nanosleep(32);
          if (++idle == 64) {
            idle_since = global_timer_ns();
          } else if (idle > 64 && (idle & 63) == 0) {
            if (*abort_flag || global_timer_ns() - idle_since > kWaitLimitNs) {
              *abort_flag = 1;
              set_status(a.status, PKV_DEV_TIMEOUT);
              break;
            }
          }
        }
      }
      // every MMA this thread issued has finished before tensor memory is freed
      umma_commit(drain);
      mbar_wait(drain, 0);
    }
    __syncwarp();
  } else {
    // ================= softmax warps (one thread per TMEM lane) =================
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m_used[N], lp[N], o_reg[N];
#pragma unroll
    for (int h = 0; h < N; ++h) m_used[h] = -INFINITY, lp[h] = 0.f, o_reg[h] = 0.f;
    bool restart = true;           // the next P·V starts a fresh TMEM accumulation
    bool pv_since_restart = false;
    int n_valid_tiles = 0;
    int obuf = 1;  // O buffer of the current item (alternates per item)
    // An item's output is written one tile later, after the next tile's P is released, so
    // its last P·V completes meanwhile instead of being waited for.
    bool fin = false;
    int4 f_mt = make_int4(0, 0, 0, 0);
    float f_o[N], f_lp[N], f_m[N];
    int f_ob = 0, f_b = 0;
    bool f_has_o = false;
    uint32_t ob_next = 0;     // bit b: parity of the phase the next P·V on o_bar[b] completes
    uint32_t ob_pending = 0;  // bit b: the last P·V on o_bar[b] has not been waited for yet
    auto wait_ob = [&](int b) -> bool {
      if (!((ob_pending >> b) & 1)) return true;
      ob_pending &= ~(1u << b);
      return mbar_wait(&o_bar[b], ((ob_next >> b) & 1) ^ 1u);
    };

    // ---- the held item's output: O = registers + TMEM, denominators, output or partial
    auto finalize = [&]() {
      fin = false;
      bool ok = true;
      float ot[N];
      if (f_has_o) {
        ok = wait_ob(f_b);  // its last P·V (the latest on P buffer f_b)
        tc_fence_after();
        float o[N];
        tmem_load_row<N>(tmem + lane_base + kColO + f_ob * 16, o);
        tc_fence_before();
#pragma unroll
        for (int h = 0; h < N; ++h) ot[h] = f_o[h] + o[h];
      } else {
#pragma unroll
        for (int h = 0; h < N; ++h) ot[h] = f_o[h];
      }
      if (!ok) *abort_flag = 1;
      float* red2 = red + 64 + f_ob * 64;  // consecutive items use different halves
      const float wsum = warp_col16<false>(f_lp, lane);
      if ((lane & 1) == 0) red2[warp * 16 + (lane >> 1)] = wsum;
      named_barrier_sync(1, kConsumers);
      const int seq = f_mt.x, kvh = f_mt.y & 0xffff, part = f_mt.z & 0xffff, nparts = f_mt.z >> 16;
      const int d = tid;
      const int64_t unit0 = static_cast<int64_t>(seq) * a.num_heads + kvh * g;
#pragma unroll
      for (int h = 0; h < N; ++h) {
        if (h >= g) break;
        const float l = red2[h] + red2[16 + h] + red2[32 + h] + red2[48 + h];
        if (nparts == 1 && !a.always_partial) {
          store_out<OUT_F32>(a, (unit0 + h) * kD + d, l > 0.f ? ot[h] / l : 0.f);
        } else {
          // unnormalised partial; a separate kernel merges the partitions
          const int64_t pidx = (unit0 + h) * a.max_parts + part;
          a.part_o[pidx * kD + d] = ot[h];
          if (d == 0) a.part_ml[pidx] = make_float2(f_m[h], l);
        }
      }
    };
    bool ended = false;

    for (int n = 0;; ++n) {
      const int slot = n % STAGES;
      bool bad = !mbar_wait(&full[slot], (n / STAGES) & 1);
      const int4 mt = meta[slot];
      if (mt.w & kMetaEnd) {
        ended = true;
        break;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      const int n_valid = mt.w & 0xff;
      const uint32_t mask = (mt.w >> 8) & 0xff;
      const bool first = mt.w & kMetaFirst, last = mt.w & kMetaLast;
      if (first) {
#pragma unroll
        for (int h = 0; h < N; ++h) m_used[h] = -INFINITY, lp[h] = 0.f, o_reg[h] = 0.f;
        restart = true;
        pv_since_restart = false;
        obuf ^= 1;
      }
      if (n_valid > 0) {
        const int b = n_valid_tiles & 1;
        unsigned char* p_tile = p_buf + b * 4096;
        bad |= !mbar_wait(&s_full[b], (n_valid_tiles >> 1) & 1);
        tc_fence_after();
        float s[N];
        tmem_load_row<N>(tmem + lane_base + b * 16, s);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[b]);
        bad |= !wait_ob(b);  // P buffer b: the P·V of two valid tiles back is done
        const int t = tid;   // this thread's row = token of the tile
        const bool valid = t < n_valid && ((mask >> (t / kChunk)) & 1);
        float x[N];
        bool need = false;
#pragma unroll
        for (int h = 0; h < N; ++h) {
          x[h] = (valid && h < g) ? s[h] * a.scale_log2 : -INFINITY;
          need |= x[h] > m_used[h] + kRescaleLog2;
        }
        // P row of this token (B operand, MN-major, unswizzled): heads 0..7 as one
        // 16-byte chunk at (t/8)*128 + (t%8)*16, heads 8..15 2 KiB further.
        float pv[N];
        auto write_p = [&]() {
          uint32_t w[N / 2];
#pragma unroll
          for (int j = 0; j < N / 2; ++j) {
            const int h0 = 2 * j, h1 = 2 * j + 1;
            const float p0 = (valid && h0 < g && m_used[h0] > -INFINITY) ? fast_exp2(x[h0] - m_used[h0]) : 0.f;
            const float p1 = (valid && h1 < g && m_used[h1] > -INFINITY) ? fast_exp2(x[h1] - m_used[h1]) : 0.f;
            w[j] = pack_bf16x2(p0, p1);
            pv[h0] = bf16lo(w[j]);
            pv[h1] = bf16hi(w[j]);
          }
          unsigned char* row = p_tile + (t >> 3) * 128 + (t & 7) * 16;
          *reinterpret_cast<uint4*>(row) = make_uint4(w[0], w[1], w[2], w[3]);
          if (g > 8) *reinterpret_cast<uint4*>(row + 2048) = make_uint4(w[4], w[5], w[6], w[7]);
        };
        if (!valid) {
          // rows of V outside the context may hold anything (even NaN): zero them
          uint4* r0 = reinterpret_cast<uint4*>(v_ring + slot * kTileBytes + t * 128);
          uint4* r1 = reinterpret_cast<uint4*>(v_ring + slot * kTileBytes + kHalfBytes + t * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) r0[c] = r1[c] = make_uint4(0, 0, 0, 0);
        }
        if (bad) *abort_flag = 1;
        bool need_any = true;  // an item's first tile always sets the held maximum
        if (!first) {
          write_p();
          if (tid == 0) restart_flag[b] = (restart ? 1 : 0) | (obuf << 1);
          fence_proxy_async_smem();
          need_any = named_barrier_or(1, kConsumers, need || bad);
          if (*abort_flag) break;
        }
        if (need_any) {
          // A score outgrew the held maximum (or none is held yet): take the tile
          // maximum, fold the accumulated P·V into registers at the old scale, and
          // (re)write P.
          const float wmax = warp_col16<true>(x, lane);
          if ((lane & 1) == 0) red[warp * 16 + (lane >> 1)] = wmax;
          bool ok = true;
          if (pv_since_restart) {  // this item's O is folded below: its P·Vs must be complete
            ok = wait_ob(0);
            ok &= wait_ob(1);
          }
          if (!ok) *abort_flag = 1;
          named_barrier_sync(1, kConsumers);
          if (*abort_flag) break;
          float alpha[N];
#pragma unroll
          for (int h = 0; h < N; ++h) {
            const float tmax = fmaxf(fmaxf(red[h], red[16 + h]), fmaxf(red[32 + h], red[48 + h]));
            if (h < g) {
              // nothing is accumulated yet while the held maximum is -inf
              const float m_new = fmaxf(m_used[h], tmax);
              alpha[h] = m_used[h] == -INFINITY ? 0.f : fast_exp2(m_used[h] - m_new);
              m_used[h] = m_new;
            } else {
              alpha[h] = 1.f;
            }
          }
          tc_fence_after();
          if (pv_since_restart) {
            float o[N];
            tmem_load_row<N>(tmem + lane_base + kColO + obuf * 16, o);
#pragma unroll
            for (int h = 0; h < N; ++h) o_reg[h] = (o_reg[h] + o[h]) * alpha[h];
          } else {
#pragma unroll
            for (int h = 0; h < N; ++h) o_reg[h] *= alpha[h];
          }
          tc_fence_before();
#pragma unroll
          for (int h = 0; h < N; ++h) lp[h] *= alpha[h];
          restart = true;
          pv_since_restart = false;
          write_p();
          if (tid == 0) restart_flag[b] = 1 | (obuf << 1);
          fence_proxy_async_smem();
          named_barrier_sync(1, kConsumers);
        }
#pragma unroll
        for (int h = 0; h < N; ++h)
          if (h < g) lp[h] += pv[h];
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
        ob_next ^= 1u << b;
        ob_pending |= 1u << b;
        restart = false;
        pv_since_restart = true;
        ++n_valid_tiles;
      }
      if (fin) finalize();  // the previous item: its last P·V ran while this tile was processed
      if (last) {
        fin = true;
        f_mt = mt;
#pragma unroll
        for (int h = 0; h < N; ++h) f_o[h] = o_reg[h], f_lp[h] = lp[h], f_m[h] = m_used[h];
        f_ob = obuf;
        f_has_o = pv_since_restart;
        f_b = (n_valid_tiles - 1) & 1;  // P buffer of the item's last valid tile
      }
    }
    if (ended && fin) finalize();
    if (*abort_flag && tid == 0) set_status(a.status, PKV_DEV_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// Merge of split partitions: one CTA of 4 warps per (sequence, query head) whose
// context was split, o = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p.  Runs
// after the main kernel on the same stream.  Warp w takes partitions w, w+4, ...;
// lane l owns output values 4l .. 4l+3; the four warps' sums meet in shared memory.
constexpr int kMergeWarps = 4;

template <bool OUT_F32>
__global__ void __launch_bounds__(kMergeWarps * 32) merge_partials_kernel(const DecodeArgs a) {
  __shared__ float s_max[kMergeWarps];
  __shared__ float s_l[kMergeWarps];
  __shared__ float4 s_acc[kMergeWarps][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int seq = blockIdx.x / a.num_heads, h = blockIdx.x % a.num_heads;
  int L = a.context_lens[seq];
  if (L < 0 || L > a.max_context_len || L > a.max_blocks * a.block_size) L = 0;  // as the plan does
  const int nparts = L == 0 ? 1 : (L + a.partition - 1) / a.partition;
  griddep_wait();  // the decode kernel has finished: its partials are visible
  if (nparts <= 1) return;  // written directly by the main kernel
  const int64_t unit = static_cast<int64_t>(seq) * a.num_heads + h;
  const float2* ml = a.part_ml + unit * a.max_parts;
  const float* po = a.part_o + unit * a.max_parts * kD + lane * 4;
  float M = -INFINITY;
  for (int p = warp + kMergeWarps * lane; p < nparts; p += kMergeWarps * 32) M = fmaxf(M, ml[p].x);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if (lane == 0) s_max[warp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(s_max[0], s_max[1]), fmaxf(s_max[2], s_max[3]));
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float Ls = 0.f;
  for (int base = warp; base < nparts; base += kMergeWarps * 32) {
    const int p = base + kMergeWarps * lane;  // this lane's partition of the round
    float w = 0.f;
    if (p < nparts) {
      const float2 v = ml[p];
      w = v.x == -INFINITY ? 0.f : exp2f(v.x - M);
      Ls = fmaf(w, v.y, Ls);
    }
    const int cnt = min(32, (nparts - base + kMergeWarps - 1) / kMergeWarps);
#pragma unroll 8
    for (int j = 0; j < cnt; ++j) {
      const float wj = __shfl_sync(0xffffffffu, w, j);
      const float4 o = *reinterpret_cast<const float4*>(po + static_cast<int64_t>(base + kMergeWarps * j) * kD);
      acc.x = fmaf(wj, o.x, acc.x);
      acc.y = fmaf(wj, o.y, acc.y);
      acc.z = fmaf(wj, o.z, acc.z);
      acc.w = fmaf(wj, o.w, acc.w);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, off);
  if (lane == 0) s_l[warp] = Ls;
  s_acc[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    const float Lt = s_l[0] + s_l[1] + s_l[2] + s_l[3];
    const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
    float4 r = s_acc[0][lane];
#pragma unroll
    for (int w2 = 1; w2 < kMergeWarps; ++w2) {
      const float4 t = s_acc[w2][lane];
      r.x += t.x, r.y += t.y, r.z += t.z, r.w += t.w;
    }
    const int64_t base = unit * kD + lane * 4;
    store_out<OUT_F32>(a, base + 0, r.x * inv);
    store_out<OUT_F32>(a, base + 1, r.y * inv);
    store_out<OUT_F32>(a, base + 2, r.z * inv);
    store_out<OUT_F32>(a, base + 3, r.w * inv);
  }
}

// ---- host side -----------------------------------------------------------

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
  static PerDevice<int> setup;
  int dev = 0, sms = 0;
  const int st = set_smem_limit_once(setup, kernel, smem, &dev);
  if (st != 0) return set_error(PKV_ERR_CUDA, "decode (tensor) setup: %s", cudaGetErrorString(static_cast<cudaError_t>(st)));
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaError_t e = launch_after_previous(kernel, dim3(std::max(1, sms)), dim3(kThreads), smem, stream, args);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "decode (tensor) launch: %s", cudaGetErrorString(e));
  return args.a.always_partial ? PKV_OK : launch_merge_partials(args.a, OUT_F32, stream);
}

}  // namespace tc

int launch_merge_partials(const DecodeArgs& a, bool out_f32, cudaStream_t stream) {
  if (a.max_parts <= 1) return PKV_OK;
  const dim3 grid(a.num_seqs * a.num_heads), block(tc::kMergeWarps * 32);
  cudaError_t e = out_f32 ? launch_after_previous(tc::merge_partials_kernel<true>, grid, block, 0, stream, a)
                          : launch_after_previous(tc::merge_partials_kernel<false>, grid, block, 0, stream, a);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "decode merge launch: %s", cudaGetErrorString(e));
  return PKV_OK;
}

bool tensor_path_supports(int group, int head_dim) { return head_dim == tc::kD && group >= 2 && group <= 16; }

int launch_decode_tensor(const DecodeArgs& a, int head_dim, bool out_f32, cudaStream_t stream) {
  if (!tensor_path_supports(a.group, head_dim))
    return set_error(PKV_ERR_UNSUPPORTED, "decode (tensor): group %d / head_dim %d not supported", a.group, head_dim);
  tc::Args args;
  args.a = a;
  constexpr int n = 16;
  const uint64_t pool_rows = static_cast<uint64_t>(a.num_blocks) * a.num_kv_heads * a.block_size;
  const uint32_t rows = static_cast<uint32_t>(tc::box_rows(a.block_size));
  int rc = tc::encode_map(&args.tm_k, a.key_cache, pool_rows, rows, "key_cache");
  if (rc == PKV_OK) rc = tc::encode_map(&args.tm_v, a.value_cache, pool_rows, rows, "value_cache");
  if (rc == PKV_OK)
    rc = tc::encode_map(&args.tm_q, a.query, static_cast<uint64_t>(a.num_seqs) * a.num_heads, n, "query");
  if (rc != PKV_OK) return rc;
  return out_f32 ? tc::launch<n, true>(args, stream) : tc::launch<n, false>(args, stream);
}

}  // namespace pkv
