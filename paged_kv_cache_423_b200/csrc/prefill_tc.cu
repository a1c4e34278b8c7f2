// Tensor-core (tcgen05) prefill / chunked-prefill attention over the paged cache.
//
// Each sequence brings n new tokens (its chunk; Outcome School explainer, "LLM
// serving的基本流程与KV缓存": prefill reads the prompt at once; intelliparadigm
// article §4.1/§4.2: chunked prefill feeds a long prompt in pieces) whose K/V are
// already in the pool.  Chunk row i is the token at position p = L - n + i and
// attends causally to positions 0 .. p, read page by page through the block table.
//
// Unlike decode, the query side is dense.  A query tile is 128 rows = 128 / g tokens
// x the g query heads of one kv head (row m = token * g + head).  A CTA holds TWO
// consecutive query tiles (A and B) of one (sequence, kv head) and streams the K/V
// pages once for both, 128 keys per stage:
//   S_t[128 x 128] = Q_t[128 x D] · K[128 x D]ᵀ     (A = Q_t in shared memory, B = K;
//                                                    both K-major, TMA-swizzled)
//   online softmax of each row (one thread per TMEM lane; causal mask on the diagonal)
//   O_t[128 x D]  += P_t[128 x 128] · V[128 x D]    (A = P_t in TENSOR memory, written
//                                                    over S_t by the softmax threads;
//                                                    B = V, MN-major)
// Shared-memory bandwidth is what bounds these MMAs: keeping P in tensor memory and
// using 128-wide S tiles leaves only Q, K and V to cross shared memory.
//
// Tensor memory (512 columns): S_t / P_t in columns t*128 .. t*128+127 (P_t, bf16,
// takes the first 64), O_t in 256 + t*128.  Per tile the MMA order is
// ... S_t(n) -> [softmax] -> O_t += P_t(n)·V(n) -> S_t(n+1) ..., so S_t(n+1) never
// overwrites P_t(n) before its P·V has read it, and once a softmax group sees S_t(n+1)
// every earlier MMA of the tile is complete (a commit covers all prior MMAs), so O_t
// may be rescaled without a further wait.  O is rescaled only when a row's maximum
// grows by more than 2^8; P is rounded to bf16 and the row sums add the same values.
//
// Work item = (pair of query tiles, kv head), from a plan ordered longest sequence
// first with every tile pair of a sequence adjacent, so items that read the same
// K/V pages run at the same time and share them through L2.  CTAs are persistent and
// take items from a counter.  Roles: warps 0-3 softmax + epilogue of tile A, warps
// 4-7 of tile B, warp 8 TMA producer (K one stage ahead of V), warp 9 MMA issuer (a
// fixed order with blocking waits).  Per-stage metadata travels in its own ring.
// Every wait is bounded; on a timeout the CTA flags PKV_DEV_TIMEOUT, lets its copies
// land, waits for its MMAs, frees its tensor memory and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "decode_common.cuh"
#include "launch_setup.cuh"
#include "pkv_internal.h"
#include "tcgen05_common.cuh"

namespace pkv {
namespace pf {

using tc::fast_exp2;

constexpr int kRows = 128;                  // query rows per tile (MMA M)
constexpr int kKeys = 128;                  // keys per stage (MMA N of S, K of P·V)
constexpr int kD = 128;                     // head_dim of this path
constexpr int kHalf = 128 * 128;            // one 64-column half of a 128-row bf16 tile: 16 KiB
constexpr int kTileBytes = 2 * kHalf;       // a Q, K or V tile: 32 KiB
constexpr int kChunk = 16;                  // key rows per TMA box (a 16-row slice of one block)
constexpr int kChunks = kKeys / kChunk;     // 8
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kMetaSlots = 8;
constexpr int kSoftmaxWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 384;              // 3 warpgroups; warps 10-11 only lend registers
// Register split (setmaxnreg): launched at 168 per thread (384 x 168 = 64512); the
// producer/MMA warpgroup drops to 120 and the two softmax warpgroups rise to 192:
// 128 x (192 + 192 + 120) = 64512 <= 64512, and per scheduler (one warp of each
// group) 32 x 504 = 16128 <= 16384 registers.  ptxas fits both roles without
// spilling at these counts (at 208 / 88 the control warps spilled).
constexpr int kRegsSoftmax = 192;
constexpr int kRegsControl = 120;
static_assert(128 * (2 * kRegsSoftmax + kRegsControl) <= kThreads * 168, "register split exceeds the launch");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr float kRescaleLog2 = 8.f;
// Share of the softmax exponentials computed by a polynomial on the FMA pipe (one pair of
// scores in kPolyEvery; 0 = none, the default).  The SFU issues 16 exponentials per clock per
// SM, about as many as a stage's MMAs take; but measured on a B200 every share made the kernel
// slower (13B chunked batch: 746 TFLOP/s with none, 677 with one pair in 8, 637 with one in 4,
// 528 with one in 2): the softmax is bound by instruction issue, and the polynomial adds
// instructions.  The option stays for other shapes; its function is tested either way.
#ifndef PKV_PREFILL_POLY_EVERY
#define PKV_PREFILL_POLY_EVERY 0
#endif
constexpr int kPolyEvery = PKV_PREFILL_POLY_EVERY;

// shared memory (offsets from a 1024-aligned base)
constexpr int kOffQ = 0;                                   // [2 tiles]
constexpr int kOffK = kOffQ + 2 * kTileBytes;              // [3 stages]
constexpr int kOffV = kOffK + kKStages * kTileBytes;       // [2 stages]
constexpr int kOffMeta = kOffV + kVStages * kTileBytes;    // [8] int4
constexpr int kOffBar = kOffMeta + kMetaSlots * 16;
constexpr int kBars = 2 + 2 * kKStages + 2 * kVStages + 2 * kMetaSlots + 2 + 2 + 2 + 1;
constexpr int kOffMisc = kOffBar + kBars * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;           // + slack to align the base
static_assert(kSmemBytes <= 232448, "shared memory of one CTA");

// Stage metadata: x = packed row of tile A's first token, y = its position,
// z = tokens of tile A | tokens of tile B << 8 | kv head << 16,
// w = stage index in the item (18 bits) | chunk mask << 18 | flags.
constexpr int kFirst = 1 << 26, kLast = 1 << 27, kEnd = 1 << 28;

struct PrefillArgs {
  void* out;
  const int32_t* block_tables;
  const int32_t* plan_count;  // [0] entries, [1] work-item counter
  const int4* entries;        // x = first packed row, y = its position, z = tokens A | tokens B << 8, w = sequence
                              // (segment mode: w = part, y unused)
  const int4* parts;          // segment mode: [2 * part] (table row, first block, keys, first row),
                              //               [2 * part + 1] (rows, first partial, first scratch block, 0)
  float* part_o;              // segment mode: unnormalised partial outputs [partial][head][128]
  float2* part_ml;            // segment mode: (held maximum in base-2 units, weight sum) [partial][head]
  int32_t* status;
  int max_blocks;
  int num_heads;
  int num_kv_heads;
  int block_size;
  int num_blocks;
  int group;
  int group_shift;            // log2(group)
  int tile_tokens;            // 128 / group
  float scale_log2;
  // segment mode over widened 8-bit blocks: per-kv-head factors of the scores and of the
  // partial outputs (the codes' scales), or null
  const float* k_scale;
  const float* v_scale;
};

struct alignas(64) Args {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  PrefillArgs a;
};

// a0 += w.lo, a1 += w.hi for the two bf16 values of w, each by fma.rn.f32.bf16 with 1 as the
// other factor: exact product, one rounding of the sum.
__device__ __forceinline__ void add_bf16x2(float& a0, float& a1, uint32_t w) {
  asm("{\n\t.reg .b16 lo, hi, one;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "mov.b16 one, 0x3F80;\n\t"
      "fma.rn.f32.bf16 %0, lo, one, %0;\n\t"
      "fma.rn.f32.bf16 %1, hi, one, %1;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(w));
}

// SEG = false: causal prefill, normalised output rows.  SEG = true: the shared phase of
// the shared-prefix decode — every query row of an item sees all keys of its part (a run
// of whole blocks of one table row), and the epilogue writes unnormalised partials.
template <bool OUT_F32, bool SEG>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ Args args) {
  const PrefillArgs& a = args.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_buf = smem + kOffQ;
  unsigned char* k_ring = smem + kOffK;
  unsigned char* v_ring = smem + kOffV;
  int4* meta = reinterpret_cast<int4*>(smem + kOffMeta);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;                        // [K stage]
  uint64_t* k_empty = k_full + kKStages;              // [K stage]
  uint64_t* v_full = k_empty + kKStages;              // [V stage]
  uint64_t* v_empty = v_full + kVStages;              // [V stage]
  uint64_t* meta_full = v_empty + kVStages;           // [meta slot]
  uint64_t* meta_free = meta_full + kMetaSlots;       // [meta slot]
  uint64_t* s_full = meta_free + kMetaSlots;          // [tile]: S_t of the stage is in tensor memory
  uint64_t* p_full = s_full + 2;                      // [tile]: P_t of the stage is in tensor memory
  uint64_t* o_bar = p_full + 2;                       // [tile]: O_t += P_t·V of the stage done
  uint64_t* drain = o_bar + 2;                        // the MMA thread's last commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = a.group;

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
    for (int s = 0; s < kMetaSlots; ++s) {
      mbar_init(&meta_full[s], 1);
      mbar_init(&meta_free[s], kSoftmaxWarps);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 4);  // one arrival per warp of the tile's group
      mbar_init(&o_bar[t], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tc::tmem_alloc(tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The set-up above overlaps the plan kernel (when launched after it); its work list is
  // read only after it has finished.
  griddep_wait();
  const int64_t n_items = static_cast<int64_t>(a.plan_count[0]) * a.num_kv_heads;
  auto fail = [&]() {
    *abort_flag = 1;
    set_status(a.status, PKV_DEV_TIMEOUT);
  };

  if (warp >= kProducerWarp) {
  // The control warpgroup gives registers back; the branch is uniform per warpgroup,
  // as setmaxnreg requires, and dominates the code that runs with the new count.
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
  if (warp == kProducerWarp) {
    // ================= producer =================
    // Stages form one stream across items.  K of stage n+1 (with its metadata) is
    // issued before V of stage n, so the QK side runs a stage ahead; at an item
    // boundary V of the old item goes first, then the new item's queries.
    const uint64_t pol_q = l2_policy_evict_first();
    const uint64_t pol_kv = l2_policy_evict_normal();  // every tile pair of the sequence re-reads these pages
    int* work_counter = const_cast<int*>(a.plan_count) + 1;
    auto grab = [&]() -> int64_t {
      int v = 0;
      if (lane == 0) v = atomicAdd(work_counter, 1);
      return __shfl_sync(0xffffffffu, v, 0);
    };
    bool failed = false;
    auto wait_slot = [&](uint64_t* bar, int fills, int depth) -> bool {
      if (failed) return false;
      // warp-uniform: every lane takes the same branch (the copies below are per lane)
      if (fills >= depth && !__all_sync(0xffffffffu, pipe_wait(bar, ((fills / depth) - 1) & 1))) {
        fail();
        failed = true;
      }
      return !failed;
    };
    // the item whose stages the K side is issuing
    int64_t item = grab();
    int kvh = 0, row0 = 0, pos0 = 0, ntok_a = 0, ntok_b = 0, nkeys = 0, nst = 0, j = 0, meta_x = 0;
    const int32_t* table = nullptr;
    int tab_cur = -1, tab_nxt = -1, win = 0;
    // Table entries come 32 slices (4 stages) at a time, one window ahead: lane l
    // holds the physical block of slice 32 w + l of window w.
    auto load_window = [&](int w) -> int {
      const int kp = (w * 32 + lane) * kChunk;
      return kp < nkeys ? __ldg(table + kp / a.block_size) : -1;
    };
    auto start_item = [&]() {
      const int4 e = a.entries[item / a.num_kv_heads];
      kvh = static_cast<int>(item % a.num_kv_heads);
      row0 = e.x;
      ntok_a = e.z & 0xff;
      ntok_b = (e.z >> 8) & 0xff;
      if constexpr (SEG) {
        // the stage metadata carries the pair's first partial id and the part's key count
        const int4 pd0 = a.parts[2 * e.w], pd1 = a.parts[2 * e.w + 1];
        nkeys = pd0.z;
        meta_x = pd1.y + (e.x - pd0.w);
        pos0 = nkeys;
        table = a.block_tables + static_cast<int64_t>(pd0.x) * a.max_blocks + pd0.y;
      } else {
        pos0 = e.y;
        nkeys = pos0 + ntok_a + ntok_b;
        meta_x = row0;
        table = a.block_tables + static_cast<int64_t>(e.w) * a.max_blocks;
      }
      nst = (nkeys + kKeys - 1) / kKeys;
      j = 0;
      win = 0;
      tab_cur = load_window(0);
      tab_nxt = load_window(1);
    };
    int kn = 0, vn = 0, q_loads = 0;  // K fills, V fills, query loads issued
    auto load_q = [&]() -> bool {
      if (q_loads > 0 && !wait_slot(q_empty, q_loads, 1)) return false;
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full, (ntok_b > 0 ? 2 : 1) * kTileBytes);
        tc::tma_load_3d(q_buf, &args.tm_q, 0, kvh * g, row0, q_full, pol_q);
        tc::tma_load_3d(q_buf + kHalf, &args.tm_q, 64, kvh * g, row0, q_full, pol_q);
        if (ntok_b > 0) {
          tc::tma_load_3d(q_buf + kTileBytes, &args.tm_q, 0, kvh * g, row0 + a.tile_tokens, q_full, pol_q);
          tc::tma_load_3d(q_buf + kTileBytes + kHalf, &args.tm_q, 64, kvh * g, row0 + a.tile_tokens, q_full, pol_q);
        }
      }
      ++q_loads;
      return true;
    };
    // K (and metadata) of the cursor's stage j; returns this lane's V source row
    // and the slice mask through the references, for the matching V fill.
    auto issue_k = [&](int& vrow, uint32_t& vmask) -> bool {
      if (j / 4 != win) {
        ++win;
        tab_cur = tab_nxt;
        tab_nxt = load_window(win + 1);
      }
      const int kbase = j * kKeys;
      const int nvalid = min(kKeys, nkeys - kbase);
      const int nch = (nvalid + kChunk - 1) / kChunk;
      const int kp = kbase + lane * kChunk;  // this lane's 16-row slice (lanes < nch)
      const bool mine = lane < nch;
      int phys = __shfl_sync(0xffffffffu, tab_cur, (j % 4) * 8 + (lane & 7));
      if (!mine) phys = -1;
      const bool ok = mine && phys >= 0 && phys < a.num_blocks;
      const uint32_t mask = __ballot_sync(0xffffffffu, ok) & 0xffu;
      if (mine && !ok) set_status(a.status, PKV_DEV_BAD_BLOCK);
      vrow = ok ? (phys * a.num_kv_heads + kvh) * a.block_size + kp % a.block_size : -1;
      vmask = mask;
      if (!wait_slot(&k_empty[kn % kKStages], kn, kKStages)) return false;
      if (!wait_slot(&meta_free[kn % kMetaSlots], kn, kMetaSlots)) return false;
      const int ks = kn % kKStages;
      if (lane == 0) {
        meta[kn % kMetaSlots] = make_int4(meta_x, pos0, ntok_a | (ntok_b << 8) | (kvh << 16),
                                          j | static_cast<int>(mask << 18) | (j == 0 ? kFirst : 0) |
                                              (j == nst - 1 ? kLast : 0));
        mbar_arrive(&meta_full[kn % kMetaSlots]);
        mbar_arrive_expect_tx(&k_full[ks], __popc(mask) * kChunk * 256);
      }
      __syncwarp();
      if (ok) {
        unsigned char* kd = k_ring + ks * kTileBytes + lane * kChunk * 128;
        tc::tma_load_2d(kd, &args.tm_k, 0, vrow, &k_full[ks], pol_kv);
        tc::tma_load_2d(kd + kHalf, &args.tm_k, 64, vrow, &k_full[ks], pol_kv);
      }
      ++kn;
      return true;
    };
    auto issue_v = [&](int vrow, uint32_t vmask) -> bool {
      if (!wait_slot(&v_empty[vn % kVStages], vn, kVStages)) return false;
      const int vs = vn % kVStages;
      if (lane == 0) mbar_arrive_expect_tx(&v_full[vs], __popc(vmask) * kChunk * 256);
      __syncwarp();
      if (vrow >= 0) {
        unsigned char* vd = v_ring + vs * kTileBytes + lane * kChunk * 128;
        tc::tma_load_2d(vd, &args.tm_v, 0, vrow, &v_full[vs], pol_kv);
        tc::tma_load_2d(vd + kHalf, &args.tm_v, 64, vrow, &v_full[vs], pol_kv);
      }
      ++vn;
      return true;
    };
    int pend_row = -1;
    uint32_t pend_mask = 0;
    bool pending = false;  // V of the last K-issued stage still to go
    if (item < n_items) {
      start_item();
      if (load_q() && issue_k(pend_row, pend_mask)) pending = true;
    }
    while (pending && !failed && !*abort_flag) {
      // advance the cursor to the next stage
      ++j;
      bool new_item = false;
      if (j == nst) {
        item = grab();
        new_item = true;
      }
      int nrow;
      uint32_t nmask;
      if (new_item) {
        if (!issue_v(pend_row, pend_mask)) break;
        pending = false;
        if (item >= n_items) break;
        start_item();
        if (!load_q() || !issue_k(pend_row, pend_mask)) break;
        pending = true;
      } else {
        if (!issue_k(nrow, nmask)) break;
        if (!issue_v(pend_row, pend_mask)) break;
        pend_row = nrow;
        pend_mask = nmask;
      }
    }
    if (!failed && !*abort_flag && wait_slot(&k_empty[kn % kKStages], kn, kKStages) &&
        wait_slot(&meta_free[kn % kMetaSlots], kn, kMetaSlots)) {
      // end-of-stream: a K fill and metadata with no data
      if (lane == 0) {
        meta[kn % kMetaSlots] = make_int4(0, 0, 0, kEnd);
        mbar_arrive(&meta_full[kn % kMetaSlots]);
        mbar_arrive_expect_tx(&k_full[kn % kKStages], 0);
      }
      ++kn;
      __syncwarp();
    }
    // Let this CTA's last copies land before the final barrier.
    for (int k = max(0, kn - kKStages); k < kn; ++k) mbar_wait(&k_full[k % kKStages], (k / kKStages) & 1);
    for (int k = max(0, vn - kVStages); k < vn; ++k) mbar_wait(&v_full[k % kVStages], (k / kVStages) & 1);
    if (q_loads > 0) mbar_wait(q_full, (q_loads - 1) & 1);
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer (one thread) =================
    // Fixed order with blocking waits, one barrier at a time:
    //   S_A(0) S_B(0) | PV_A(0) S_A(1) PV_B(0) S_B(1) | PV_A(1) S_A(2) ...
    // P·V of a tile goes before its next S (P lives in S's columns), and the other
    // tile's MMAs fill the tensor pipe while one group runs its softmax.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc::instr_desc(kRows, kKeys, false, false);
      constexpr uint32_t idesc_pv = tc::instr_desc(kRows, kD, false, true);
      int sc[2] = {0, 0}, pc[2] = {0, 0};  // per tile: S and P·V issued
      int q_items = 0;
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        if (ok && !pipe_wait(bar, parity)) {
          ok = false;
          fail();
        }
        return ok;
      };
      auto stage_meta = [&](int n) -> int4 { return meta[n % kMetaSlots]; };
      auto has_b = [](const int4& mt) { return ((mt.z >> 8) & 0xff) != 0; };
      // S_t = Q_t·Kᵀ of stage n (K landed, queries of a new item landed).
      auto issue_s = [&](int n, int t, const int4& mt) -> bool {
        if (t == 0 && (mt.w & kFirst)) {
          if (!wait(q_full, q_items & 1)) return false;
          ++q_items;
        }
        tc::tc_fence_after();
        const uint32_t q_addr = smem_addr(q_buf + t * kTileBytes);
        const uint32_t k_addr = smem_addr(k_ring + (n % kKStages) * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          tc::umma(tmem + t * 128, tc::smem_desc_sw128(q_addr + off, 16, 1024),
                   tc::smem_desc_sw128(k_addr + off, 16, 1024), idesc_qk, kk > 0);
        }
        tc::umma_commit(&s_full[t]);
        ++sc[t];
        const bool stage_done = t == 1 || !has_b(mt);
        if (stage_done) {
          tc::umma_commit(&k_empty[n % kKStages]);
          if (mt.w & kLast) tc::umma_commit(q_empty);
        }
        return true;
      };
      // O_t += P_t·V of stage n (P in tensor memory, V landed).
      auto issue_pv = [&](int n, int t, const int4& mt) -> bool {
        if (t == 0 && !wait(&v_full[n % kVStages], (n / kVStages) & 1)) return false;
        if (!wait(&p_full[t], pc[t] & 1)) return false;
        tc::tc_fence_after();
        const uint32_t v_addr = smem_addr(v_ring + (n % kVStages) * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          // P: 8 columns (16 keys) per step; V: MN-major, 16 key rows per step
          tc::umma_ts(tmem + kColO + t * 128, tmem + t * 128 + kk * 8,
                      tc::smem_desc_sw128(v_addr + kk * 2048, kHalf, 1024), idesc_pv,
                      kk > 0 || !(mt.w & kFirst));
        }
        tc::umma_commit(&o_bar[t]);
        ++pc[t];
        if (t == 1 || !has_b(mt)) tc::umma_commit(&v_empty[n % kVStages]);
        return true;
      };
      // stage 0
      bool more = wait(&k_full[0], 0) && !(stage_meta(0).w & kEnd);
      if (more) {
        const int4 m0 = stage_meta(0);
        more = issue_s(0, 0, m0) && (!has_b(m0) || issue_s(0, 1, m0));
      }
      for (int n = 0; more && ok; ++n) {
        const int4 mt = stage_meta(n);
        // the next stage's K (or the end marker)
        if (!wait(&k_full[(n + 1) % kKStages], ((n + 1) / kKStages) & 1)) break;
        const int4 mn = stage_meta(n + 1);
        const bool next = !(mn.w & kEnd);
        if (next && !(mn.w & kFirst)) {
          // same item: interleave per tile
          if (!issue_pv(n, 0, mt) || !issue_s(n + 1, 0, mn)) break;
          if (has_b(mt) && !issue_pv(n, 1, mt)) break;
          if (has_b(mn) && !issue_s(n + 1, 1, mn)) break;
        } else {
          // item boundary or end: finish this item's P·V first
          if (!issue_pv(n, 0, mt)) break;
          if (has_b(mt) && !issue_pv(n, 1, mt)) break;
          if (!next) break;
          if (!issue_s(n + 1, 0, mn)) break;
          if (has_b(mn) && !issue_s(n + 1, 1, mn)) break;
        }
      }
      // every MMA this thread issued has finished before tensor memory is freed
      tc::umma_commit(drain);
      mbar_wait(drain, 0);
    }
    __syncwarp();
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ================= softmax warps: thread = query row of tile t = TMEM lane =================
    const int t = warp >> 2;                 // 0: tile A (warps 0-3), 1: tile B (warps 4-7)
    const int m = tid & 127;                 // row within the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t col_s = t * 128, col_o = kColO + t * 128;
    float m_used = -INFINITY, lsum = 0.f;
    float sl2 = a.scale_log2;  // score scale (base 2) of the item; segment mode may fold in the key scale
    bool has_pv = false;
    int c = 0;  // stages of this tile processed (phases of s_full / p_full / o_bar)
    for (int n = 0;; ++n) {
      bool ok = __all_sync(0xffffffffu, pipe_wait(&meta_full[n % kMetaSlots], (n / kMetaSlots) & 1));
      const int4 mt = meta[n % kMetaSlots];
      __syncwarp();
      if (lane == 0) mbar_arrive(&meta_free[n % kMetaSlots]);
      if (!ok || (mt.w & kEnd)) {  // warp-uniform: every lane leaves together
        if (!ok) *abort_flag = 1;
        break;
      }
      const int ntok_a = mt.z & 0xff, ntok_b = (mt.z >> 8) & 0xff, kvh = mt.z >> 16;
      const int ntok = t == 0 ? ntok_a : ntok_b;
      if (ntok == 0) continue;  // tile B absent from this item
      const int j = mt.w & 0x3ffff;
      const uint32_t mask = (mt.w >> 18) & 0xffu;
      const bool first = mt.w & kFirst, last = mt.w & kLast;
      // causal: row0 = packed row, pos0 = its position; segment mode: row0 = partial id, mt.y = keys
      const int row0 = mt.x + t * a.tile_tokens, pos0 = mt.y + t * a.tile_tokens;
      if (first) {
        m_used = -INFINITY;
        lsum = 0.f;
        has_pv = false;
        if constexpr (SEG) sl2 = a.k_scale ? a.scale_log2 * __ldg(a.k_scale + kvh) : a.scale_log2;
      }
      const int tl = m >> a.group_shift;
      const bool valid_row = tl < ntok;
      const int limit = SEG ? mt.y - 1 : pos0 + (valid_row ? tl : ntok - 1);  // last visible key position
      const int kbase = j * kKeys;
      const int nvalid = min(kKeys, (SEG ? mt.y : mt.y + ntok_a + ntok_b) - kbase);
      if (t == 0 && (nvalid < kKeys || mask != 0xffu)) {
        // V rows past the context or in a slice that was not loaded may hold anything
        // (even NaN): zero them once the stage's copies have landed, before P·V.
        const int vs = n % kVStages;
        ok &= pipe_wait(&v_full[vs], (n / kVStages) & 1);
        if (m >= nvalid || !((mask >> (m / kChunk)) & 1u)) {
          unsigned char* vrow = v_ring + vs * kTileBytes + m * 128;
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 8; ++q) reinterpret_cast<uint4*>(vrow + h * kHalf)[q] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      // ---- S row (its arrival also means every earlier MMA of this tile is done)
      ok &= pipe_wait(&s_full[t], c & 1);
      tc::tc_fence_after();
      float s[kKeys];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) tc::tmem_load32f_nowait(tmem + lane_base + col_s + q4 * 32, s + q4 * 32);
      tc::tmem_wait_ld();
      // ---- causal / context mask and the row maximum
      if (!(kbase + kKeys - 1 <= (SEG ? mt.y - 1 : pos0) && mask == 0xffu)) {
#pragma unroll
        for (int k = 0; k < kKeys; ++k) {
          const bool vis = kbase + k <= limit && ((mask >> (k / kChunk)) & 1u);
          s[k] = vis ? s[k] : -INFINITY;
        }
      }
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = s[i];
#pragma unroll
      for (int k = 8; k < kKeys; ++k) mx8[k & 7] = fmaxf(mx8[k & 7], s[k]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float mxs = mx * sl2;
      // A row rescales only when its maximum grew past the threshold; the tensor-memory
      // accesses are warp-collective, so the warp rescales together (alpha = 1 for the
      // rows that keep their maximum).  Every P·V of the tile is complete here.
      const bool need = mxs > m_used + kRescaleLog2;
      float alpha = 1.f;
      if (need) {
        const float m_new = fmaxf(m_used, mxs);
        alpha = m_used == -INFINITY ? 0.f : fast_exp2(m_used - m_new);
        m_used = m_new;
      }
      if (has_pv && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t r[32];
          tc::tmem_load32_nowait(tmem + lane_base + col_o + q4 * 32, r);
          tc::tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
          tc::tmem_store32(tmem + lane_base + col_o + q4 * 32, r);
        }
      }
      lsum *= alpha;
      // ---- P = 2^(s * scale_log2 - m) as bf16 pairs, stored over S (columns 0-63 of
      //      the tile's block: keys 2i, 2i+1 in column i).  Pairs of scores go through packed
      //      fp32x2 arithmetic: one fma.rn.f32x2 for scale and maximum.  The row sum adds the
      //      rounded bf16 values into eight fp32 accumulators with the mixed-precision FMA
      //      (x·1 + acc: one rounding, the same sum as an fp32 add of the widened value,
      //      without widening it first).  A row with no visible key yet holds -inf as its
      //      maximum: neg_m is then 0 and every score of the stage is -inf, so its weights
      //      are 0 without a select.
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      const uint64_t sc2 = f2pack(sl2, sl2), nm2 = f2pack(neg_m, neg_m);
      float ls[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) ls[i] = 0.f;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 e = f2unpack(ffma2(f2pack(s[h * 32 + 2 * i], s[h * 32 + 2 * i + 1]), sc2, nm2));
          // one pair in kPolyEvery takes the FMA-pipe exponential, the rest the SFU's
          const bool poly = kPolyEvery > 0 && (i % kPolyEvery) == kPolyEvery - 1;
          const float p0 = poly ? tc::poly_exp2(e.x) : fast_exp2(e.x);
          const float p1 = poly ? tc::poly_exp2(e.y) : fast_exp2(e.y);
          w[i] = pack_bf16x2(p0, p1);
          add_bf16x2(ls[2 * (i & 3)], ls[2 * (i & 3) + 1], w[i]);
        }
        tc::tmem_store16(tmem + lane_base + col_s + h * 16, w);
      }
      {
        const float l0x = ls[0] + ls[2], l0y = ls[1] + ls[3], l1x = ls[4] + ls[6], l1y = ls[5] + ls[7];
        lsum += (l0x + l0y) + (l1x + l1y);
      }
      tc::tmem_wait_st();
      tc::tc_fence_before();     // P and the rescaled O, before the MMA reads them
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
      has_pv = true;
      ++c;
      if (last) {
        // ---- epilogue: O / l of this row, once the item's last P·V is done
        ok &= pipe_wait(&o_bar[t], (c - 1) & 1);
        tc::tc_fence_after();
        const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
        const int64_t orow = (static_cast<int64_t>(row0 + tl) * a.num_heads + kvh * g + (m & (g - 1))) * kD;
        float vsc = 1.f;  // segment mode over widened 8-bit blocks: the value scale of the kv head
        if constexpr (SEG) {
          if (valid_row) a.part_ml[orow / kD] = make_float2(m_used, lsum);
          if (a.v_scale) vsc = __ldg(a.v_scale + kvh);
        }
        uint32_t r[32];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          tc::tmem_load32_nowait(tmem + lane_base + col_o + q4 * 32, r);
          tc::tmem_wait_ld();
          if (valid_row) {
            if constexpr (SEG) {
              float4* dst = reinterpret_cast<float4*>(a.part_o + orow + q4 * 32);
#pragma unroll
              for (int k = 0; k < 8; ++k)
                dst[k] = make_float4(__uint_as_float(r[4 * k]) * vsc, __uint_as_float(r[4 * k + 1]) * vsc,
                                     __uint_as_float(r[4 * k + 2]) * vsc, __uint_as_float(r[4 * k + 3]) * vsc);
            } else if constexpr (OUT_F32) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow + q4 * 32);
#pragma unroll
              for (int k = 0; k < 8; ++k)
                dst[k] = make_float4(__uint_as_float(r[4 * k]) * inv, __uint_as_float(r[4 * k + 1]) * inv,
                                     __uint_as_float(r[4 * k + 2]) * inv, __uint_as_float(r[4 * k + 3]) * inv);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + orow + q4 * 32);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint32_t* v = r + 8 * k;
                dst[k] = make_uint4(pack_bf16x2(__uint_as_float(v[0]) * inv, __uint_as_float(v[1]) * inv),
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
    if (*abort_flag && (tid & 127) == 0) set_status(a.status, PKV_DEV_TIMEOUT);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

// ---- plan ---------------------------------------------------------------------
//
// One CTA.  Validates every sequence, then lays the query-tile pairs out longest
// sequence first (counting sort on the context length, coarsened to 512 buckets),
// each sequence's pairs adjacent and its longest pair first.  A sequence whose
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
  griddep_launch_dependents();  // the prefill kernel may be scheduled now; it waits for this one to end
  for (int i = threadIdx.x; i < kPlanBuckets; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  const int pair_tokens = 2 * p.tile_tokens;
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
    if (n > 0) atomicAdd(&cnt[plan_bucket(L, p.max_context_len)], (n + pair_tokens - 1) / pair_tokens);
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
    const int npairs = (n + pair_tokens - 1) / pair_tokens;
    const int pos = atomicAdd(&cnt[plan_bucket(L, p.max_context_len)], npairs);
    for (int k = 0; k < npairs; ++k) {
      const int pair = npairs - 1 - k;  // longest (last) pair first
      const int t0 = pair * pair_tokens;
      const int na = min(p.tile_tokens, n - t0);
      const int nb = max(0, min(p.tile_tokens, n - t0 - p.tile_tokens));
      p.entries[pos + k] = make_int4(q0 + t0, L - n + t0, na | (nb << 8), s);
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

// after_plan: launched right after the plan kernel on the same stream, chained to it (the
// shared-prefix decode's segment launch follows an event wait on its side stream instead).
template <bool OUT_F32, bool SEG = false>
static int launch_main(const Args& args, int grid, cudaStream_t stream, bool after_plan) {
  auto kernel = prefill_tc_kernel<OUT_F32, SEG>;
  static PerDevice<int> setup;
  int dev = 0;
  const int st = set_smem_limit_once(setup, kernel, kSmemBytes, &dev);
  if (st != 0) return set_error(PKV_ERR_CUDA, "prefill setup: %s", cudaGetErrorString(static_cast<cudaError_t>(st)));
  cudaError_t e = cudaSuccess;
  if (after_plan)
    e = launch_after_previous(kernel, dim3(grid), dim3(kThreads), kSmemBytes, stream, args);
  else
    kernel<<<grid, kThreads, kSmemBytes, stream>>>(args);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e));
  return PKV_OK;
}

// Plan entries the workspace must hold: one per pair of query tiles.
static int max_entries(int num_seqs, int total_q, int group) {
  const int pair_tokens = 2 * (kRows / group);
  return (total_q + pair_tokens - 1) / pair_tokens + num_seqs;
}

}  // namespace pf

int launch_prefill_segments(const SegmentLaunch& L, cudaStream_t s) {
  const int group = L.num_heads / L.num_kv_heads;
  pf::Args args;
  pf::PrefillArgs& a = args.a;
  a.out = nullptr;
  a.block_tables = L.block_tables;
  a.plan_count = L.plan_count;
  a.entries = L.entries;
  a.parts = L.parts;
  a.part_o = L.part_o;
  a.part_ml = L.part_ml;
  a.status = L.status;
  a.max_blocks = L.max_blocks;
  a.num_heads = L.num_heads;
  a.num_kv_heads = L.num_kv_heads;
  a.block_size = L.block_size;
  a.num_blocks = L.num_blocks;
  a.group = group;
  a.group_shift = __builtin_ctz(static_cast<unsigned>(group));
  a.tile_tokens = pf::kRows / group;
  a.scale_log2 = L.scale * 1.4426950408889634f;
  a.k_scale = L.k_scale;
  a.v_scale = L.v_scale;
  const uint64_t pool_rows = static_cast<uint64_t>(L.num_blocks) * L.num_kv_heads * L.block_size;
  int rc = pf::encode_kv_map(&args.tm_k, L.key_cache, pool_rows, "key_cache");
  if (rc == PKV_OK) rc = pf::encode_kv_map(&args.tm_v, L.value_cache, pool_rows, "value_cache");
  if (rc == PKV_OK) rc = pf::encode_q_map(&args.tm_q, L.query, L.num_seqs, L.num_heads, group);
  if (rc != PKV_OK) return rc;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t items = static_cast<int64_t>(L.num_entries) * L.num_kv_heads;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(sms, items)));
  return pf::launch_main<true, true>(args, grid, s, false);
}

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
  if (num_kv_heads >= (1 << 15) || max_context_len >= (1 << 25))
    return set_error(PKV_ERR_INVALID, "paged_attention_prefill: sizes out of range");
  if (!(scale > 0.f) || !std::isfinite(scale))  // masked keys are -inf scores: a scale of 0 would make them NaN
    return set_error(PKV_ERR_INVALID, "paged_attention_prefill: scale must be finite and positive");
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
  a.tile_tokens = pf::kRows / group;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.k_scale = nullptr;
  a.v_scale = nullptr;
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
  return p.out_f32 ? pf::launch_main<true, false>(args, grid, s, true) : pf::launch_main<false, false>(args, grid, s, true);
}
