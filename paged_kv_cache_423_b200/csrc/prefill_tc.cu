// Tensor-core (tcgen05) prefill / chunked-prefill attention over the paged cache.
//
// Each sequence brings n new tokens (its chunk; Outcome School explainer, "LLM
// serving的基本流程与KV缓存": prefill reads the prompt at once; intelliparadigm
// article §4.1/§4.2: chunked prefill feeds a long prompt in pieces) whose K/V are
// already in the pool.  Chunk row i is the token at position p = L - n + i and
// attends causally to positions 0 .. p, read page by page through the block table.
//
// Unlike decode, the query side is dense: a tile is 128 query rows = 128 / g tokens
// x the g query heads of one kv head (row m = token * g + head), and every K/V tile
// is shared by all of them.  Per 128-key tile:
//   S[128 x 128] = Q[128 x D] · K[128 x D]ᵀ       (A = Q, B = K; both K-major, TMA-swizzled)
//   online softmax of each row (one thread per TMEM lane; causal mask on the diagonal)
//   O[128 x D]  += P[128 x 128] · V[128 x D]      (A = P, K-major, written by the softmax
//                                                   threads; B = V, MN-major)
// S is double-buffered in tensor memory (columns 0-127, 128-255), O lives in columns
// 256-383 for the whole item.  O is rescaled in tensor memory only when a row's
// maximum grows by more than 2^8; P is rounded to bf16 for the MMA and the row sums
// add the same rounded values.
//
// Work item = (query tile, kv head), from a plan ordered longest sequence first with
// every tile of a sequence adjacent, so the tiles that read the same K/V pages run
// at the same time and share them through L2.  CTAs are persistent and take items
// from a counter.  Roles: warps 0-3 softmax + epilogue, warp 4 TMA producer, warp 5
// MMA issuer.  Every wait is bounded; on a timeout the CTA flags PKV_DEV_TIMEOUT,
// lets its copies land, frees its tensor memory and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "decode_common.cuh"
#include "pkv_internal.h"
#include "tcgen05_common.cuh"

namespace pkv {
namespace pf {

using tc::fast_exp2;

constexpr int kRows = 128;                // query rows per tile (MMA M)
constexpr int kKeys = 128;                // keys per tile
constexpr int kD = 128;                   // head_dim of this path
constexpr int kHalf = 128 * 128;          // one 64-column half of a 128-row bf16 tile: 16 KiB
constexpr int kTileBytes = 2 * kHalf;
constexpr int kChunk = 16;                // key rows per TMA box (a 16-row slice of one block)
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr float kRescaleLog2 = 8.f;

// shared memory (offsets from a 1024-aligned base)
constexpr int kOffQ = 0;
constexpr int kOffP = kOffQ + kTileBytes;
constexpr int kOffK = kOffP + kTileBytes;
constexpr int kOffV = kOffK + kKStages * kTileBytes;
constexpr int kOffMetaV = kOffV + kVStages * kTileBytes;
constexpr int kOffMetaK = kOffMetaV + kVStages * 16;
constexpr int kOffBar = kOffMetaK + 16;
constexpr int kBars = 19;
constexpr int kOffMisc = kOffBar + kBars * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack to align the base

// V-slot metadata: x = packed row of the tile's first token, y = its position,
// z = tokens in the tile | kv head << 8, w = key tile | chunk mask << 20 | flags.
constexpr int kFirst = 1 << 28, kLast = 1 << 29, kEnd = 1 << 30;

struct PrefillArgs {
  void* out;
  const int32_t* block_tables;
  const int32_t* plan_count;  // [0] entries, [1] work-item counter
  const int4* entries;        // x = first packed row, y = its position, z = tokens, w = sequence
  int32_t* status;
  int max_blocks;
  int num_heads;
  int num_kv_heads;
  int block_size;
  int num_blocks;
  int group;
  int group_shift;            // log2(group)
  float scale_log2;
};

struct alignas(64) Args {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  PrefillArgs a;
};

template <bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ Args args) {
  const PrefillArgs& a = args.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_buf = smem + kOffQ;
  unsigned char* p_buf = smem + kOffP;
  unsigned char* k_ring = smem + kOffK;
  unsigned char* v_ring = smem + kOffV;
  int4* meta_v = reinterpret_cast<int4*>(smem + kOffMetaV);
  int* meta_k = reinterpret_cast<int*>(smem + kOffMetaK);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;   // [3]
  uint64_t* k_empty = bars + 5;  // [3]
  uint64_t* v_full = bars + 8;   // [2]
  uint64_t* v_empty = bars + 10; // [2]
  uint64_t* s_full = bars + 12;  // [2]
  uint64_t* s_free = bars + 14;  // [2]
  uint64_t* p_full = bars + 16;
  uint64_t* o_bar = bars + 17;
  uint64_t* drain = bars + 18;   // the MMA thread's last commit, before tensor memory is freed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = a.group;
  const int64_t n_items = static_cast<int64_t>(a.plan_count[0]) * a.num_kv_heads;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 4);  // one arrival per softmax warp
    }
    mbar_init(p_full, 4);
    mbar_init(o_bar, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tc::tmem_alloc(tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    // ================= producer =================
    const uint64_t pol_q = l2_policy_evict_first();
    const uint64_t pol_kv = l2_policy_evict_normal();  // every query tile of the sequence re-reads these pages
    int* work_counter = const_cast<int*>(a.plan_count) + 1;
    auto grab = [&]() -> int64_t {
      int v = 0;
      if (lane == 0) v = atomicAdd(work_counter, 1);
      return __shfl_sync(0xffffffffu, v, 0);
    };
    auto acquire = [&](uint64_t* bar, int fills, int stages) -> bool {
      if (fills >= stages && !mbar_wait(bar, ((fills / stages) - 1) & 1)) {
        *abort_flag = 1;
        set_status(a.status, PKV_DEV_TIMEOUT);
        return false;
      }
      return true;
    };
    int kn = 0, vn = 0, item_ord = 0, q_loads = 0;
    bool failed = false;
    for (int64_t item = grab(); item < n_items && !failed && !*abort_flag; item = grab(), ++item_ord) {
      const int4 e = a.entries[item / a.num_kv_heads];
      const int kvh = static_cast<int>(item % a.num_kv_heads);
      const int row0 = e.x, pos0 = e.y, ntok = e.z, seq = e.w;
      const int nkeys = pos0 + ntok;
      const int nkt = (nkeys + kKeys - 1) / kKeys;
      // Q: the previous item's last S = Q·Kᵀ must be done with the buffer
      if (item_ord > 0 && !mbar_wait(q_empty, (item_ord - 1) & 1)) {
        *abort_flag = 1;
        set_status(a.status, PKV_DEV_TIMEOUT);
        failed = true;
        break;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full, kTileBytes);
        tc::tma_load_3d(q_buf, &args.tm_q, 0, kvh * g, row0, q_full, pol_q);
        tc::tma_load_3d(q_buf + kHalf, &args.tm_q, 64, kvh * g, row0, q_full, pol_q);
      }
      ++q_loads;
      const int32_t* table = a.block_tables + static_cast<int64_t>(seq) * a.max_blocks;
      for (int j = 0; j < nkt; ++j) {
        const int kbase = j * kKeys;
        const int nvalid = min(kKeys, nkeys - kbase);
        const int nch = (nvalid + kChunk - 1) / kChunk;
        const int kp = kbase + lane * kChunk;  // this lane's 16-row slice (lanes < nch)
        const bool mine = lane < nch;
        int phys = -1;
        if (mine) phys = __ldg(table + kp / a.block_size);
        const bool ok = mine && phys >= 0 && phys < a.num_blocks;
        const uint32_t mask = __ballot_sync(0xffffffffu, ok) & 0xffu;
        if (mine && !ok) set_status(a.status, PKV_DEV_BAD_BLOCK);
        const int row = (phys * a.num_kv_heads + kvh) * a.block_size + kp % a.block_size;
        const int flags = (j == 0 ? kFirst : 0) | (j == nkt - 1 ? kLast : 0);
        // K
        const int ks = kn % kKStages;
        if (!acquire(&k_empty[ks], kn, kKStages)) {
          failed = true;
          break;
        }
        if (lane == 0) {
          meta_k[ks] = flags;
          mbar_arrive_expect_tx(&k_full[ks], __popc(mask) * kChunk * 256);
        }
        __syncwarp();
        if (ok) {
          unsigned char* kd = k_ring + ks * kTileBytes + lane * kChunk * 128;
          tc::tma_load_2d(kd, &args.tm_k, 0, row, &k_full[ks], pol_kv);
          tc::tma_load_2d(kd + kHalf, &args.tm_k, 64, row, &k_full[ks], pol_kv);
        }
        ++kn;
        // V
        const int vs = vn % kVStages;
        if (!acquire(&v_empty[vs], vn, kVStages)) {
          failed = true;
          break;
        }
        if (lane == 0) {
          meta_v[vs] = make_int4(row0, pos0, ntok | (kvh << 8), j | static_cast<int>(mask << 20) | flags);
          mbar_arrive_expect_tx(&v_full[vs], __popc(mask) * kChunk * 256);
        }
        __syncwarp();
        if (ok) {
          unsigned char* vd = v_ring + vs * kTileBytes + lane * kChunk * 128;
          tc::tma_load_2d(vd, &args.tm_v, 0, row, &v_full[vs], pol_kv);
          tc::tma_load_2d(vd + kHalf, &args.tm_v, 64, row, &v_full[vs], pol_kv);
        }
        ++vn;
      }
    }
    if (!failed && !*abort_flag) {
      // end-of-stream markers: fills with no data
      const int ks = kn % kKStages, vs = vn % kVStages;
      if (acquire(&k_empty[ks], kn, kKStages)) {
        if (lane == 0) {
          meta_k[ks] = kEnd;
          mbar_arrive_expect_tx(&k_full[ks], 0);
        }
        ++kn;
        if (acquire(&v_empty[vs], vn, kVStages)) {
          if (lane == 0) {
            meta_v[vs] = make_int4(0, 0, 0, kEnd);
            mbar_arrive_expect_tx(&v_full[vs], 0);
          }
          ++vn;
        }
      }
      __syncwarp();
    }
    // Let this CTA's last copies land before the final barrier.
    for (int k = max(0, kn - kKStages); k < kn; ++k) mbar_wait(&k_full[k % kKStages], (k / kKStages) & 1);
    for (int k = max(0, vn - kVStages); k < vn; ++k) mbar_wait(&v_full[k % kVStages], (k / kVStages) & 1);
    if (q_loads > 0) mbar_wait(q_full, (q_loads - 1) & 1);
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer (one thread) =================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc::instr_desc(kRows, kKeys, false, false);
      constexpr uint32_t idesc_pv = tc::instr_desc(kRows, kD, false, true);
      const uint32_t q_addr = smem_addr(q_buf);
      const uint32_t p_addr = smem_addr(p_buf);
      int qn = 0, pn = 0, end_n = 0x7fffffff, q_items = 0;
      bool q_ready = false;
      uint64_t idle_since = 0;
      int idle = 0;
      while (pn < end_n) {
        bool progress = false;
        // ---- S = Q·Kᵀ of the next landed key tile
        if (qn < end_n && mbar_test(&k_full[qn % kKStages], (qn / kKStages) & 1)) {
          const int f = meta_k[qn % kKStages];
          if (f & kEnd) {
            end_n = qn;
            progress = true;
          } else {
            if ((f & kFirst) && !q_ready) {
              q_ready = mbar_test(q_full, q_items & 1);
              if (q_ready) ++q_items;
            }
            const int b = qn & 1;
            if (q_ready && (qn < 2 || mbar_test(&s_free[b], ((qn >> 1) - 1) & 1))) {
              tc::tc_fence_after();
              const uint32_t k_addr = smem_addr(k_ring + (qn % kKStages) * kTileBytes);
#pragma unroll
              for (int kk = 0; kk < kD / 16; ++kk) {
                const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
                tc::umma(tmem + b * kKeys, tc::smem_desc_sw128(q_addr + off, 16, 1024),
                         tc::smem_desc_sw128(k_addr + off, 16, 1024), idesc_qk, kk > 0);
              }
              tc::umma_commit(&s_full[b]);
              tc::umma_commit(&k_empty[qn % kKStages]);
              if (f & kLast) {
                tc::umma_commit(q_empty);
                q_ready = false;
              }
              ++qn;
              progress = true;
            }
          }
        }
        // ---- O += P·V of the oldest tile whose P is ready
        if (pn < qn && mbar_test(p_full, pn & 1) && mbar_test(&v_full[pn % kVStages], (pn / kVStages) & 1)) {
          const int vs = pn % kVStages;
          const int w = meta_v[vs].w;  // the softmax warps waited for this fill before arriving
          tc::tc_fence_after();
          const uint32_t v_addr = smem_addr(v_ring + vs * kTileBytes);
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk) {
            // P: K-major, 128-byte swizzle (as TMA writes it); V: MN-major, 16 key rows per step
            tc::umma(tmem + kColO, tc::smem_desc_sw128(p_addr + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024),
                     tc::smem_desc_sw128(v_addr + kk * 2048, kHalf, 1024), idesc_pv, kk > 0 || !(w & kFirst));
          }
          tc::umma_commit(o_bar);
          tc::umma_commit(&v_empty[vs]);
          ++pn;
          progress = true;
        }
        if (progress) {
          idle = 0;
        } else {
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
      tc::umma_commit(drain);
      mbar_wait(drain, 0);
    }
    __syncwarp();
  } else {
    // ================= softmax warps: thread = query row = TMEM lane =================
    const int m = tid;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m_used = -INFINITY, lsum = 0.f;
    bool has_pv = false;
    int waited_pv = 0;  // P·V completions this thread has observed
    for (int t = 0;; ++t) {
      const int vs = t % kVStages;
      bool ok = __all_sync(0xffffffffu, mbar_wait(&v_full[vs], (t / kVStages) & 1));
      const int4 mt = meta_v[vs];
      if (!ok || (mt.w & kEnd)) {  // warp-uniform: every lane leaves together
        if (!ok) *abort_flag = 1;
        break;
      }
      const int j = mt.w & 0xfffff;
      const uint32_t mask = (mt.w >> 20) & 0xffu;
      const bool first = mt.w & kFirst, last = mt.w & kLast;
      const int row0 = mt.x, pos0 = mt.y, ntok = mt.z & 0xff, kvh = mt.z >> 8;
      if (first) {
        m_used = -INFINITY;
        lsum = 0.f;
        has_pv = false;
      }
      const int tl = m >> a.group_shift;
      const bool valid_row = tl < ntok;
      const int limit = pos0 + (valid_row ? tl : ntok - 1);  // last visible key position
      const int kbase = j * kKeys;
      const int nvalid = min(kKeys, pos0 + ntok - kbase);
      // V rows past the context or in a slice that was not loaded may hold anything
      // (even NaN): zero them before P·V reads the tile.
      if (m >= nvalid || !((mask >> (m / kChunk)) & 1u)) {
        uint4* r0 = reinterpret_cast<uint4*>(v_ring + vs * kTileBytes + m * 128);
        uint4* r1 = reinterpret_cast<uint4*>(v_ring + vs * kTileBytes + kHalf + m * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) r0[c] = r1[c] = make_uint4(0, 0, 0, 0);
      }
      // ---- S row
      const int b = t & 1;
      ok = mbar_wait(&s_full[b], (t >> 1) & 1);
      tc::tc_fence_after();
      float s[kKeys];
      {
        uint32_t r[32];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          tc::tmem_load32_nowait(tmem + lane_base + b * kKeys + q4 * 32, r);
          tc::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) s[q4 * 32 + c] = __uint_as_float(r[c]);
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[b]);
      // ---- causal / context mask and the row maximum
      const bool full_tile = kbase + kKeys - 1 <= pos0 && mask == 0xffu;
      if (!full_tile) {
#pragma unroll
        for (int c = 0; c < kKeys; ++c) {
          const bool vis = kbase + c <= limit && ((mask >> (c / kChunk)) & 1u);
          s[c] = vis ? s[c] : -INFINITY;
        }
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < kKeys; ++c) mx = fmaxf(mx, s[c]);
      const float mxs = mx * a.scale_log2;
      // The single P buffer and O: the previous tile's P·V must be done.
      if (t > waited_pv) {
        ok &= mbar_wait(o_bar, (t - 1) & 1);
        waited_pv = t;
      }
      // A row rescales only when its maximum grew past the threshold; the tensor-memory
      // accesses are warp-collective, so the warp rescales together (alpha = 1 for
      // the rows that keep their maximum).
      const bool need = mxs > m_used + kRescaleLog2;
      float alpha = 1.f;
      if (need) {
        const float m_new = fmaxf(m_used, mxs);
        alpha = m_used == -INFINITY ? 0.f : fast_exp2(m_used - m_new);
        m_used = m_new;
      }
      if (has_pv && __any_sync(0xffffffffu, need)) {
        tc::tc_fence_after();
        uint32_t r[32];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          tc::tmem_load32_nowait(tmem + lane_base + kColO + q4 * 32, r);
          tc::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * alpha);
          tc::tmem_store32(tmem + lane_base + kColO + q4 * 32, r);
        }
        tc::tmem_wait_st();
      }
      lsum *= alpha;
      // ---- P = 2^(s * scale_log2 - m), bf16, written as the K-major swizzled A operand
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      const bool any = m_used != -INFINITY;
      unsigned char* prow = p_buf + m * 128;
#pragma unroll
      for (int c8 = 0; c8 < kKeys / 8; ++c8) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float x0 = s[c8 * 8 + 2 * i], x1 = s[c8 * 8 + 2 * i + 1];
          const float p0 = any ? fast_exp2(fmaf(x0, a.scale_log2, neg_m)) : 0.f;
          const float p1 = any ? fast_exp2(fmaf(x1, a.scale_log2, neg_m)) : 0.f;
          w[i] = pack_bf16x2(p0, p1);
          lsum += bf16lo(w[i]) + bf16hi(w[i]);
        }
        const int half = c8 >> 3, chunk = c8 & 7;
        *reinterpret_cast<uint4*>(prow + half * kHalf + ((chunk ^ (m & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();  // P and the zeroed V rows, before the MMA reads them
      tc::tc_fence_before();     // the rescaled O, before the next P·V
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      has_pv = true;
      if (last) {
        // ---- epilogue: O / l of this row
        ok &= mbar_wait(o_bar, t & 1);
        waited_pv = t + 1;
        tc::tc_fence_after();
        const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
        const int64_t orow = (static_cast<int64_t>(row0 + tl) * a.num_heads + kvh * g + (m & (g - 1))) * kD;
        uint32_t r[32];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          tc::tmem_load32_nowait(tmem + lane_base + kColO + q4 * 32, r);
          tc::tmem_wait_ld();
          if (valid_row) {
            if constexpr (OUT_F32) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow + q4 * 32);
#pragma unroll
              for (int c = 0; c < 8; ++c)
                dst[c] = make_float4(__uint_as_float(r[4 * c]) * inv, __uint_as_float(r[4 * c + 1]) * inv,
                                     __uint_as_float(r[4 * c + 2]) * inv, __uint_as_float(r[4 * c + 3]) * inv);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + orow + q4 * 32);
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const uint32_t* v = r + 8 * c;
                dst[c] = make_uint4(pack_bf16x2(__uint_as_float(v[0]) * inv, __uint_as_float(v[1]) * inv),
                                    pack_bf16x2(__uint_as_float(v[2]) * inv, __uint_as_float(v[3]) * inv),
                                    pack_bf16x2(__uint_as_float(v[4]) * inv, __uint_as_float(v[5]) * inv),
                                    pack_bf16x2(__uint_as_float(v[6]) * inv, __uint_as_float(v[7]) * inv));
              }
            }
          }
        }
        tc::tc_fence_before();
      }
      if (!ok) *abort_flag = 1;
      if (__any_sync(0xffffffffu, !ok || *abort_flag)) break;  // warp-uniform
    }
    if (*abort_flag && tid == 0) set_status(a.status, PKV_DEV_TIMEOUT);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

// ---- plan ---------------------------------------------------------------------
//
// One CTA.  Validates every sequence, then lays the query tiles out longest
// sequence first (counting sort on the context length, coarsened to 512 buckets),
// each sequence's tiles adjacent and its longest tile first.  A sequence whose
// numbers are inconsistent is flagged PKV_DEV_BAD_CONTEXT and its rows, when their
// range is itself valid, are written as zeros.
constexpr int kPlanThreads = 1024;

struct PlanArgs {
  const int32_t* query_start;
  const int32_t* context_lens;
  int4* entries;
  int32_t* plan_count;
  void* out;
  int32_t* status;
  int num_seqs;
  int total_q;
  int max_context_len;
  int max_tokens;  // max_blocks * block_size
  int tile_tokens;
  int num_heads;
  int capacity;    // entries the workspace holds
  bool out_f32;
};

__device__ __forceinline__ int plan_bucket(int len, int max_len) {
  const int b = static_cast<int>((static_cast<int64_t>(max_len - len) * (kPlanBuckets - 1)) / max(max_len, 1));
  return min(max(b, 0), kPlanBuckets - 1);
}

__global__ void __launch_bounds__(kPlanThreads) prefill_plan_kernel(const PlanArgs p) {
  __shared__ int cnt[kPlanBuckets];
  __shared__ int total;
  for (int i = threadIdx.x; i < kPlanBuckets; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  auto check = [&](int s, int& q0, int& n, int& L) -> bool {
    q0 = p.query_start[s];
    const int q1 = p.query_start[s + 1];
    n = q1 - q0;
    L = p.context_lens[s];
    return q0 >= 0 && n >= 0 && q1 <= p.total_q && L >= n && L <= p.max_context_len && L <= p.max_tokens;
  };
  for (int s = threadIdx.x; s < p.num_seqs; s += blockDim.x) {
    int q0, n, L;
    if (!check(s, q0, n, L)) {
      set_status(p.status, PKV_DEV_BAD_CONTEXT);
      const int q1 = p.query_start[s + 1];
      if (q0 >= 0 && q0 <= q1 && q1 <= p.total_q) {
        const int64_t e0 = static_cast<int64_t>(q0) * p.num_heads * kD, e1 = static_cast<int64_t>(q1) * p.num_heads * kD;
        for (int64_t i = e0; i < e1; ++i) {
          if (p.out_f32)
            static_cast<float*>(p.out)[i] = 0.f;
          else
            static_cast<__nv_bfloat16*>(p.out)[i] = __float2bfloat16_rn(0.f);
        }
      }
      continue;
    }
    if (n > 0) atomicAdd(&cnt[plan_bucket(L, p.max_context_len)], (n + p.tile_tokens - 1) / p.tile_tokens);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int i = 0; i < kPlanBuckets; ++i) {
      const int c = cnt[i];
      cnt[i] = run;
      run += c;
    }
    total = run;
  }
  __syncthreads();
  if (total > p.capacity) {
    // overlapping row ranges (query_start not non-decreasing): refuse the whole call
    if (threadIdx.x == 0) {
      set_status(p.status, PKV_DEV_BAD_CONTEXT);
      p.plan_count[0] = 0;
      p.plan_count[1] = 0;
    }
    return;
  }
  for (int s = threadIdx.x; s < p.num_seqs; s += blockDim.x) {
    int q0, n, L;
    if (!check(s, q0, n, L) || n == 0) continue;
    const int ntiles = (n + p.tile_tokens - 1) / p.tile_tokens;
    const int pos = atomicAdd(&cnt[plan_bucket(L, p.max_context_len)], ntiles);
    for (int k = 0; k < ntiles; ++k) {
      const int tile = ntiles - 1 - k;  // longest (last) tile first
      const int t0 = tile * p.tile_tokens;
      p.entries[pos + k] = make_int4(q0 + t0, L - n + t0, min(p.tile_tokens, n - t0), s);
    }
  }
  if (threadIdx.x == 0) {
    p.plan_count[0] = total;
    p.plan_count[1] = 0;
  }
}

// ---- host side -----------------------------------------------------------------

static int encode_kv_map(CUtensorMap* map, const void* base, uint64_t rows, const char* what) {
  auto encode = tc::tensor_map_encoder();
  if (!encode) return set_error(PKV_ERR_CUDA, "prefill: cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), rows};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kChunk)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(PKV_ERR_CUDA, "prefill: tensor map for %s failed (%d)", what, (int)r);
  return PKV_OK;
}

// Query [T, Hq, 128] as a 3-D map (dim, head, token); box 64 x g x 128/g = one tile
// of 128 rows (token-major, heads inside), 128-byte swizzle.
static int encode_q_map(CUtensorMap* map, const void* base, int total_q, int num_heads, int group) {
  auto encode = tc::tensor_map_encoder();
  if (!encode) return set_error(PKV_ERR_CUDA, "prefill: cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(num_heads),
                        static_cast<cuuint64_t>(total_q)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD) * 2, static_cast<cuuint64_t>(num_heads) * kD * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(kRows / group)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(PKV_ERR_CUDA, "prefill: tensor map for query failed (%d)", (int)r);
  return PKV_OK;
}

template <bool OUT_F32>
static int launch_main(const Args& args, int grid, cudaStream_t stream) {
  auto kernel = prefill_tc_kernel<OUT_F32>;
  static std::once_flag once;
  static cudaError_t setup = cudaSuccess;
  std::call_once(once,
                 [&] { setup = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes); });
  if (setup != cudaSuccess) return set_error(PKV_ERR_CUDA, "prefill setup: %s", cudaGetErrorString(setup));
  kernel<<<grid, kThreads, kSmemBytes, stream>>>(args);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e));
  return PKV_OK;
}

static int max_entries(int num_seqs, int total_q, int group) {
  const int tile_tokens = kRows / group;
  return (total_q + tile_tokens - 1) / tile_tokens + num_seqs;
}

}  // namespace pf
}  // namespace pkv

using namespace pkv;

extern "C" size_t pkv_paged_attention_prefill_workspace_size(int num_seqs, int total_q, int num_heads,
                                                             int num_kv_heads) {
  if (num_seqs < 0 || total_q < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0) return 0;
  const int group = num_heads / num_kv_heads;
  if (group > pf::kRows || pf::kRows % group != 0) return 0;
  return 256 + align256(static_cast<size_t>(pf::max_entries(num_seqs, total_q, group)) * sizeof(int4));
}

extern "C" int pkv_paged_attention_prefill(void* out, int out_dtype, const void* query, const void* key_cache,
                                           const void* value_cache, const int32_t* block_tables,
                                           int max_blocks_per_seq, const int32_t* query_start,
                                           const int32_t* context_lens, int num_seqs, int total_q,
                                           int max_context_len, int num_heads, int num_kv_heads, int head_dim,
                                           int block_size, int num_blocks, float scale, void* workspace,
                                           size_t workspace_bytes, int32_t* status, pkv_stream_t stream) {
  clear_error();
  if (num_seqs < 0 || total_q < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
      max_blocks_per_seq <= 0 || max_context_len < 0)
    return set_error(PKV_ERR_INVALID, "paged_attention_prefill: bad sizes");
  if (out_dtype != PKV_DTYPE_BF16 && out_dtype != PKV_DTYPE_F32)
    return set_error(PKV_ERR_INVALID, "paged_attention_prefill: out_dtype %d", out_dtype);
  if (head_dim != pf::kD)
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_prefill: head_dim %d (only 128)", head_dim);
  if (block_size != 16 && block_size != 32)
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_prefill: block_size %d not in {16,32}", block_size);
  if (num_heads % num_kv_heads != 0)
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_prefill: num_heads %d not a multiple of num_kv_heads %d",
                     num_heads, num_kv_heads);
  const int group = num_heads / num_kv_heads;
  if (group > pf::kRows || pf::kRows % group != 0)
    return set_error(PKV_ERR_UNSUPPORTED, "paged_attention_prefill: group %d does not divide 128", group);
  if (num_kv_heads >= (1 << 23) || max_context_len >= (1 << 27))
    return set_error(PKV_ERR_INVALID, "paged_attention_prefill: sizes out of range");
  if (static_cast<int64_t>(num_blocks) * num_kv_heads * block_size > (static_cast<int64_t>(1) << 31))
    return set_error(PKV_ERR_INVALID, "paged_attention_prefill: pool too large");
  if (num_seqs == 0 || total_q == 0) return PKV_OK;
  if (static_cast<int64_t>(pf::max_entries(num_seqs, total_q, group)) * num_kv_heads > (int64_t{1} << 30))
    return set_error(PKV_ERR_INVALID, "paged_attention_prefill: too many query tiles");
  if (!out || !query || !key_cache || !value_cache || !block_tables || !query_start || !context_lens || !workspace)
    return set_error(PKV_ERR_INVALID, "paged_attention_prefill: null pointer");
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache))
    return set_error(PKV_ERR_INVALID, "paged_attention_prefill: tensors must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return set_error(PKV_ERR_INVALID, "paged_attention_prefill: workspace must be 256-byte aligned");
  const size_t need = pkv_paged_attention_prefill_workspace_size(num_seqs, total_q, num_heads, num_kv_heads);
  if (workspace_bytes < need)
    return set_error(PKV_ERR_INVALID, "paged_attention_prefill: workspace of %zu bytes, %zu needed", workspace_bytes,
                     need);

  unsigned char* ws = static_cast<unsigned char*>(workspace);
  int32_t* plan_count = reinterpret_cast<int32_t*>(ws);
  int4* entries = reinterpret_cast<int4*>(ws + 256);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  pf::PlanArgs p{};
  p.query_start = query_start;
  p.context_lens = context_lens;
  p.entries = entries;
  p.plan_count = plan_count;
  p.out = out;
  p.status = status;
  p.num_seqs = num_seqs;
  p.total_q = total_q;
  p.max_context_len = max_context_len;
  p.max_tokens = max_blocks_per_seq * block_size;
  p.tile_tokens = pf::kRows / group;
  p.num_heads = num_heads;
  p.capacity = pf::max_entries(num_seqs, total_q, group);
  p.out_f32 = out_dtype == PKV_DTYPE_F32;
  pf::prefill_plan_kernel<<<1, pf::kPlanThreads, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "prefill plan launch: %s", cudaGetErrorString(e));

  pf::Args args;
  pf::PrefillArgs& a = args.a;
  a.out = out;
  a.block_tables = block_tables;
  a.plan_count = plan_count;
  a.entries = entries;
  a.status = status;
  a.max_blocks = max_blocks_per_seq;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.group = group;
  a.group_shift = __builtin_ctz(static_cast<unsigned>(group));
  a.scale_log2 = scale * 1.4426950408889634f;
  const uint64_t pool_rows = static_cast<uint64_t>(num_blocks) * num_kv_heads * block_size;
  int rc = pf::encode_kv_map(&args.tm_k, key_cache, pool_rows, "key_cache");
  if (rc == PKV_OK) rc = pf::encode_kv_map(&args.tm_v, value_cache, pool_rows, "value_cache");
  if (rc == PKV_OK) rc = pf::encode_q_map(&args.tm_q, query, total_q, num_heads, group);
  if (rc != PKV_OK) return rc;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t items = static_cast<int64_t>(pf::max_entries(num_seqs, total_q, group)) * num_kv_heads;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(sms, items)));
  return p.out_f32 ? pf::launch_main<true>(args, grid, s) : pf::launch_main<false>(args, grid, s);
}
