// Tensor-core (tcgen05) decode over an 8-bit (e4m3) pool for grouped query heads.
//
// The contraction of the bf16 tensor-core decode (S = K·Qᵀ over 128-token tiles,
// online softmax of the g query heads of a kv head, O = Vᵀ·P; intelliparadigm
// article "PagedAttention：操作系统分页思想的跨界创新" §2.1), over a pool that holds
// e4m3 codes with one float32 scale per kv head.  Both products run as kind::f8f6f4
// MMAs straight from the e4m3 K and V tiles that TMA staged (128-byte swizzled):
//
//   S = K·Qᵀ   A = K (K-major).  B = the queries as two e4m3 terms, q·2^e = hi + lo,
//              with a power of two 2^e per head that puts the head's largest |q| in
//              [128, 256): hi is q·2^e rounded to e4m3 and lo the exact remainder
//              rounded to e4m3, which holds all 8 significant bits of a bf16 value
//              down to 2^-2 (below that the error is at most 2^-10 · 2^-e).  [hi; lo]
//              is one N = 32 operand; the softmax adds the two halves of S.
//   O = Vᵀ·P   A = V (MN-major: a token row of 128 codes is one swizzle span).  B = P
//              (times 2^7) as three e5m2 terms: hi and mid are the f16 value of P cut
//              to e5m2 and lo the rest rounded to e5m2, about 9 significant bits, and
//              e5m2's range keeps every weight above 2^-23 of the held maximum (e4m3
//              would drop those below 2^-9).  [hi | mid | lo] is one N = 48 operand;
//              the softmax adds the three thirds of O, and the denominators add the
//              same represented values.
//   The K scale and 2^-e join the score scale, the V scale the output.
//
// The queries are split into their e4m3 terms once per call, before the main kernel,
// by split_queries_kernel (one warp per (sequence, kv head)), into the workspace; the
// producer loads an item's split rows and head scales with its first tile, so no MMA
// waits for a split.  Roles: warps 0-7 softmax (two groups; thread = TMEM lane = token
// row of a tile), warp 8 TMA producer, warp 9 MMA issuer (fixed order: S of tile n+1,
// then O += Vᵀ·P of tile n).  Work items, plan, workspace and the merge of split
// partitions are those of the bf16 decode paths.
// Every wait is bounded; on a timeout the CTA flags PKV_DEV_TIMEOUT, lets its copies
// land, waits for its MMAs, frees its tensor memory and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "decode_common.cuh"
#include "launch_setup.cuh"
#include "pkv_internal.h"
#include "tcgen05_common.cuh"

namespace pkv {
namespace tc8 {

using tc::fast_exp2;

constexpr int kTile = 128;                 // tokens per tile (MMA M of S)
constexpr int kChunk = 16;                 // rows per validity bit (and per TMA box at block size 16)
constexpr int kD = 128;
constexpr int kN = 16;                     // query heads of one kv head (g <= 16)
constexpr int kRow8 = kD;                  // bytes of one e4m3 row
constexpr int kTile8 = kTile * kRow8;      // one K or V tile: 16 KiB
constexpr int kQSlot = 4096;               // e4m3 [hi; lo] queries: 32 rows x 128 codes (from the split kernel)
constexpr int kPTerm = kTile * 16;         // one e5m2 term of P: 128 tokens x 16 heads
constexpr int kPBytes = 3 * kPTerm;        // [hi | mid | lo]
constexpr uint32_t kTmemCols = 256;        // S double buffer [0,32), [32,64) (hi | lo); O of even / odd items
constexpr uint32_t kColO = 64;             // at [64,112) / [128,176) (3 terms of 16 heads each)
constexpr uint32_t kOStride = 64;
constexpr float kRescaleLog2 = 8.f;
constexpr float kPShift = 7.f;             // P is stored times 2^7 (at most 2^15)
// Stage metadata: x = sequence, y = kv head | q slot << 16, z = partition | partitions << 16,
// w = valid rows (8 bits) | slice mask << 8 | first << 16 | last << 17 | end of stream << 18
constexpr int kMetaFirst = 1 << 16, kMetaLast = 1 << 17, kMetaEnd = 1 << 18;

// Rows per TMA box: 32 where every 32-row slice stays inside one block, else 16 (the TMA
// engine's time per box limits a producer warp, so the larger box is used where it can be).
__host__ __device__ constexpr int box_rows(int block_size) { return block_size % 32 == 0 ? 32 : kChunk; }

// K and V of a tile travel in separate rings: a K slot is free again once the tile's S = K·Qᵀ
// is done, a V slot only once its O += Vᵀ·P is, so K (and with it the next tiles' S) runs a
// stage further ahead than a shared K+V stage would allow.
// Two shapes of the CTA.
//   GROUPS = 2: one CTA per SM; two softmax warpgroups split each tile's head pairs
//     (warps 0-7), warp 8 the TMA producer, warp 9 the MMA issuer, warps 10-11 only lend
//     registers; 5 K and 4 V slots.  Registers: launched at 168 per thread (384 x 168 = 64512), the
//     control warpgroup drops to 88 and the softmax warpgroups rise to 208:
//     128 x (208 + 208 + 88) = 64512, and per scheduler (one warp of each group)
//     32 x 504 = 16128 <= 16384.
//   GROUPS = 1: two CTAs per SM, so two independent item streams (each CTA's
//     MMA -> softmax -> MMA chain) overlap on one SM; one softmax warpgroup takes every head
//     (warps 0-3), warp 4 the producer, warp 5 the MMA issuer, warps 6-7 lend registers;
//     3 K and 2 V slots each.  Registers: launched at 128 (2 x 256 x 128 = 65536), softmax 184,
//     control 72: 128 x (184 + 72) = 32768 per CTA, and per scheduler 2 CTAs x 32 x 256 =
//     16384.
#ifndef PKV_FP8_K2
#define PKV_FP8_K2 5
#endif
#ifndef PKV_FP8_V2
#define PKV_FP8_V2 4
#endif
template <int GROUPS>
struct Cfg {
  static constexpr int kKStages = GROUPS == 2 ? PKV_FP8_K2 : 3;
  static constexpr int kVStages = GROUPS == 2 ? PKV_FP8_V2 : 2;
  static constexpr int kQSlots = kKStages + 1;  // by item ordinal; a slot is refilled kQSlots items later
  static constexpr int kSoftmax = 128 * GROUPS;
  static constexpr int kProducerWarp = 4 * GROUPS;
  static constexpr int kMmaWarp = 4 * GROUPS + 1;
  static constexpr int kThreads = 128 * (GROUPS + 1);
  static constexpr int kCtasPerSm = GROUPS == 2 ? 1 : 2;
  static constexpr int kLaunchRegs = GROUPS == 2 ? 168 : 128;
  static constexpr int kRegsSoftmax = GROUPS == 2 ? 208 : 184;
  static constexpr int kRegsControl = GROUPS == 2 ? 88 : 72;
  static_assert(128 * (GROUPS * kRegsSoftmax + kRegsControl) <= kThreads * kLaunchRegs,
                "register split exceeds the launch");
  static_assert(kThreads * kLaunchRegs * kCtasPerSm <= 65536, "registers of an SM");
  // shared memory
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kKStages * kTile8;
  static constexpr int kOffQ = kOffV + kVStages * kTile8;
  static constexpr int kOffP = kOffQ + kQSlots * kQSlot;
  static constexpr int kOffRed = kOffP + 2 * kPBytes;
  static constexpr int kOffMeta = kOffRed + 2 * 3 * 4 * 16 * 4;  // [group][maxima | sums of even | odd items][4 warps][16]
  static constexpr int kOffScale = kOffMeta + kKStages * 16;  // [K slot] (k_scale, v_scale) of the item
  static constexpr int kOffQinv = (kOffScale + kKStages * 8 + 15) / 16 * 16;  // [q slot][16] 2^-e of each head
  static constexpr int kOffBar = kOffQinv + kQSlots * 16 * 4;
  static constexpr int kBars = 2 * kKStages + 2 * kVStages + 2 * 4 + 1;
  static constexpr int kOffMisc = kOffBar + kBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 32 + 1024;
  static_assert(kOffBar % 8 == 0 && kOffMeta % 16 == 0 && kOffQ % 1024 == 0 && kOffQinv % 16 == 0, "alignment");
  static_assert((kSmemBytes + 1024) * kCtasPerSm <= 233472, "shared memory of an SM (1 KiB reserved per CTA)");
};

// Head slots (NH = 4, 8 or 16 >= g) served with one softmax warpgroup per CTA and two CTAs per
// SM (GROUPS = 1); larger groups take the two-warpgroup CTA.  Measured on a B200 (e4m3 pools):
// the long-context batch (g = 8) 3,440 against 3,350 GB/s, the shared-prompt batch (g = 4) 660
// against 552 GB/s of distinct bytes.
#ifndef PKV_FP8_ONE_GROUP_MAX_NH
#define PKV_FP8_ONE_GROUP_MAX_NH 8
#endif

struct alignas(64) Args {
  CUtensorMap tm_k;  // e4m3 pool as [rows, 128] bytes, box 128 x 16, 128-byte swizzle
  CUtensorMap tm_v;
  CUtensorMap tm_q;  // split e4m3 queries as [units * 32, 128] bytes, box 128 x 32, 128-byte swizzle
  DecodeArgs a;
};

// Two floats -> two e4m3 codes (round to nearest even, saturating), x0 in the low byte.
__device__ __forceinline__ uint32_t e4m3x2_rn(float x0, float x1) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(x1), "f"(x0));
  return r;
}

// Two e4m3 codes (low byte first) -> their values as f16x2 (exact).
__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t codes) {
  uint32_t r;
  asm("{\n\t.reg .b16 l;\n\tcvt.u16.u32 l, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\t}" : "=r"(r) : "r"(codes));
  return r;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint32_t sub_f16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t add_f16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ float f16lo(uint32_t w) {
  float r;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, l;\n\t}" : "=f"(r) : "r"(w));
  return r;
}

__device__ __forceinline__ float f16hi(uint32_t w) {
  float r;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.f32.f16 %0, h;\n\t}" : "=f"(r) : "r"(w));
  return r;
}

// hi + lo split of two scaled query values: the e4m3 codes of hi in the low 16 bits
// and of lo in the high 16 bits, x0's code in the low byte of each.
__device__ __forceinline__ uint32_t split_q2(float x0, float x1) {
  const uint32_t h = e4m3x2_rn(x0, x1);
  const uint32_t hf = e4m3x2_f16x2(h);
  const uint32_t l = e4m3x2_rn(x0 - f16lo(hf), x1 - f16hi(hf));
  return h | (l << 16);
}

// Three e5m2 terms of two non-negative f16 values p (f16x2): hi and mid are p cut to
// the top byte (an e5m2 code is the top byte of an f16) and lo the remainder rounded
// at its third significant bit.  Returns the three f16x2 words whose top bytes are
// the codes; `sum` gets hi + mid + lo (exact in f16).
__device__ __forceinline__ void split_p2(uint32_t p, uint32_t& hi, uint32_t& mid, uint32_t& lo, uint32_t& sum) {
  hi = p & 0xFF00FF00u;
  const uint32_t r1 = sub_f16x2(p, hi);
  mid = r1 & 0xFF00FF00u;
  const uint32_t r2 = sub_f16x2(r1, mid);
  lo = (r2 + 0x00800080u) & 0xFF00FF00u;
  sum = add_f16x2(add_f16x2(hi, mid), lo);
}

template <bool OUT_F32>
__device__ __forceinline__ void store_out(const DecodeArgs& a, int64_t idx, float v) {
  if constexpr (OUT_F32)
    static_cast<float*>(a.out)[idx] = v;
  else
    static_cast<__nv_bfloat16*>(a.out)[idx] = __float2bfloat16_rn(v);
}

// Pipeline (per CTA, persistent over work items; n counts tiles):
//   producer     -> k_full[n % K]  : K of tile n (and an item's split queries and head scales
//                                    on its first tile), with the tile's metadata
//   producer     -> v_full[n % V]  : V of tile n, issued after the K of tile n+1
//   MMA          -> s_full[b]      : S of the b-th valid tile (mod 2) in TMEM
//   softmax      -> s_free[b]      : that S read
//   softmax      -> p_full[b]      : P of that tile in shared buffer b (and its stale V rows zeroed)
//   MMA          -> o_bar[b]       : its O += Vᵀ·P done (P buffer b reusable)
//   MMA + softmax -> k_empty[n % K] : K slot done with: its S complete (commit; a plain arrival
//                    for a tile with no rows), metadata read by every softmax warp
//   MMA          -> v_empty[n % V] : V slot done with: its O += Vᵀ·P complete (commit; a plain
//                    arrival for a tile with no rows)
// Each tile's heads are split between the two softmax groups; they take every
// decision that touches the shared O accumulator (a rescale restarts it) together.
// NH (4, 8 or 16 >= g) bounds the heads the softmax works on; the operand layouts
// keep 16 head slots.
template <bool OUT_F32, int NH, int GROUPS>
__global__ void __launch_bounds__(Cfg<GROUPS>::kThreads, Cfg<GROUPS>::kCtasPerSm)
    decode_gqa_tc_fp8_kernel(const __grid_constant__ Args args) {
  using C = Cfg<GROUPS>;
  constexpr int kKStages = C::kKStages, kVStages = C::kVStages, kQSlots = C::kQSlots, kSoftmax = C::kSoftmax;
  constexpr int kProducerWarp = C::kProducerWarp, kMmaWarp = C::kMmaWarp;
  constexpr int kOffK = C::kOffK, kOffV = C::kOffV, kOffQ = C::kOffQ, kOffP = C::kOffP, kOffRed = C::kOffRed;
  constexpr int kOffMeta = C::kOffMeta, kOffScale = C::kOffScale, kOffQinv = C::kOffQinv, kOffBar = C::kOffBar;
  constexpr int kOffMisc = C::kOffMisc;
  const DecodeArgs& a = args.a;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* k_ring = smem + kOffK;
  unsigned char* v_ring = smem + kOffV;
  unsigned char* q_ring = smem + kOffQ;
  unsigned char* p_buf = smem + kOffP;
  float* red = reinterpret_cast<float*>(smem + kOffRed);
  int4* meta = reinterpret_cast<int4*>(smem + kOffMeta);
  float2* mscale = reinterpret_cast<float2*>(smem + kOffScale);
  float* qinv = reinterpret_cast<float*>(smem + kOffQinv);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* k_full = bars;                 // [K slot]: K (and on an item's first tile its queries) landed
  uint64_t* k_empty = k_full + kKStages;   // [K slot]: S done with K, metadata read by the softmax warps
  uint64_t* v_full = k_empty + kKStages;   // [V slot]: V landed
  uint64_t* v_empty = v_full + kVStages;   // [V slot]: O += Vᵀ·P done with V
  uint64_t* s_full = v_empty + kVStages;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_bar = p_full + 2;
  uint64_t* drain = o_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  // [P buffer]: bit 0 = the P·V starts a fresh accumulation, bit 1 = O buffer of the item
  volatile int* restart_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = a.group;
  griddep_launch_dependents();  // the merge kernel may be scheduled now; it waits for this one to end

  if (tid == 0) {
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1 + 4 * GROUPS);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 4 * GROUPS);
      mbar_init(&p_full[b], 4 * GROUPS);
      mbar_init(&o_bar[b], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // P bytes of head pairs from NH / 2 on are never written: they stay zero.
  for (int i = tid; i < 2 * kPBytes / 16; i += blockDim.x) reinterpret_cast<uint4*>(p_buf)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 0) tc::tmem_alloc(tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The set-up above overlaps the kernels before this one (plan, query split); the work list
  // and the split queries are read only after they have finished.
  griddep_wait();
  const int64_t n_items = static_cast<int64_t>(a.plan_count[0]) * a.num_kv_heads;

  if (warp >= kProducerWarp) {
  // The control warpgroup gives registers back; the branch is uniform per warpgroup,
  // as setmaxnreg requires, and dominates the code that runs with the new count.
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kRegsControl));
  if (warp == kProducerWarp) {
    // ================= producer: e4m3 slices and an item's queries =================
    const uint64_t policy = l2_policy_kv();
    auto load_entry = [&](int64_t it) -> PlanEntry {
      return it < n_items ? a.entries[it / a.num_kv_heads] : make_int4(0, 0, 0, 0);
    };
    // The item's block-table slice: lane l holds entries l, l+32, l+64, l+96 (an item
    // spans at most 2048 tokens = 128 blocks of 16).
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
    auto load_scales = [&](int64_t it) -> float2 {
      if (it >= n_items) return make_float2(0.f, 0.f);
      const int kvh = static_cast<int>(it % a.num_kv_heads);
      return make_float2(__ldg(a.k_scale + kvh), __ldg(a.v_scale + kvh));
    };
    int* work_counter = const_cast<int*>(a.plan_count) + 1;
    auto grab = [&]() -> int64_t {
      int v = 0;
      if (lane == 0) v = atomicAdd(work_counter, 1);
      return __shfl_sync(0xffffffffu, v, 0);
    };
    // The next item is claimed when the current one's last tile is issued, as in the bf16
    // kernel: a claimed item waits for this CTA alone.
    int64_t item = grab();
    int64_t item_nxt = n_items;
    PlanEntry e_cur = load_entry(item);
    int4 tab_cur = item < n_items ? load_tab(e_cur) : make_int4(0, 0, 0, 0);
    float2 sc_cur = load_scales(item);
    const int crow = box_rows(a.block_size);
    // Tile n's K (with its metadata, and an item's queries on its first tile) goes out before
    // tile n-1's V, so the S side runs a tile ahead of the V side.  Each lane remembers its V
    // slice (source row, or -1) of the last K-issued tile for that V fill.
    int n = 0, vn = 0, item_ord = 0;  // K fills and V fills issued
    bool failed = false;
    auto acquire = [&](uint64_t* empty_bar, int fills, int depth) -> bool {
      // warp-uniform: the copies below are per lane
      if (fills >= depth && !__all_sync(0xffffffffu, mbar_wait(&empty_bar[fills % depth], ((fills / depth) - 1) & 1))) {
        *abort_flag = 1;
        set_status(a.status, PKV_DEV_TIMEOUT);
        return false;
      }
      return true;
    };
    int pend_row = -1;
    uint32_t pend_boxes = 0;
    bool pending = false;  // the V of the last K-issued tile is still to go
    auto issue_v = [&]() -> bool {
      if (!acquire(v_empty, vn, kVStages)) return false;
      const int vs = vn % kVStages;
      if (lane == 0) mbar_arrive_expect_tx(&v_full[vs], __popc(pend_boxes) * static_cast<uint32_t>(crow * kRow8));
      __syncwarp();
      if (pend_row >= 0)
        tc::tma_load_2d(v_ring + vs * kTile8 + lane * crow * kRow8, &args.tm_v, 0, pend_row, &v_full[vs], policy);
      ++vn;
      pending = false;
      return true;
    };
    while (item < n_items && !failed && !*abort_flag) {
      const PlanEntry e = e_cur;
      const int kvh = static_cast<int>(item % a.num_kv_heads);
      const int ntok = e.w == 0 ? 0 : min(a.partition, e.w - e.y * a.partition);
      const int ntiles = ntok == 0 ? 1 : (ntok + kTile - 1) / kTile;
      const int qslot = item_ord % kQSlots;
      for (int tile = 0; tile < ntiles; ++tile, ++n) {
        const int slot = n % kKStages;
        if (tile == ntiles - 1) item_nxt = grab();
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
        if (!acquire(k_empty, n, kKStages)) {
          failed = true;
          break;
        }
        const bool with_q = tile == 0 && ntok > 0;
        if (lane == 0) {
          meta[slot] = make_int4(e.x, kvh | (qslot << 16), e.y | (e.z << 16),
                                 n_valid | (mask << 8) | (tile == 0 ? kMetaFirst : 0) |
                                     (tile == ntiles - 1 ? kMetaLast : 0));
          mscale[slot] = sc_cur;
          mbar_arrive_expect_tx(&k_full[slot],
                                __popc(boxes) * static_cast<uint32_t>(crow * kRow8) + (with_q ? kQSlot + 16 * 4 : 0));
        }
        __syncwarp();
        const int r = ok ? (phys * a.num_kv_heads + kvh) * a.block_size + ltok % a.block_size : -1;
        if (ok) tc::tma_load_2d(k_ring + slot * kTile8 + lane * crow * kRow8, &args.tm_k, 0, r, &k_full[slot], policy);
        if (with_q && lane == 0) {
          const int64_t unit = static_cast<int64_t>(e.x) * a.num_kv_heads + kvh;
          tc::tma_load_2d(q_ring + qslot * kQSlot, &args.tm_q, 0, static_cast<int>(unit * 32), &k_full[slot], policy);
          bulk_copy_g2s(qinv + qslot * 16, a.q_inv + unit * 16, 16 * 4, &k_full[slot], policy);
        }
        // then the previous tile's V
        if (pending && !issue_v()) {
          failed = true;
          ++n;
          break;
        }
        pend_row = r;
        pend_boxes = boxes;
        pending = true;
      }
      item = item_nxt;
      ++item_ord;
      e_cur = load_entry(item);
      tab_cur = item < n_items ? load_tab(e_cur) : make_int4(0, 0, 0, 0);
      sc_cur = load_scales(item);
    }
    if (!failed && !*abort_flag && pending && !issue_v()) failed = true;
    if (!failed && !*abort_flag) {
      // end of stream: a K fill with no data
      const int slot = n % kKStages;
      if (acquire(k_empty, n, kKStages)) {
        if (lane == 0) {
          meta[slot] = make_int4(0, 0, 0, kMetaEnd);
          mbar_arrive_expect_tx(&k_full[slot], 0);
        }
        ++n;
      }
      __syncwarp();
    }
    // Let this CTA's last copies land before the final barrier.
    for (int k = max(0, n - kKStages); k < n; ++k) mbar_wait(&k_full[k % kKStages], (k / kKStages) & 1);
    for (int k = max(0, vn - kVStages); k < vn; ++k) mbar_wait(&v_full[k % kVStages], (k / kVStages) & 1);
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer (one thread) =================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc::instr_desc_e4m3(kTile, 2 * kN);
      // A = V e4m3 MN-major, B = P e5m2 (format 1) MN-major, N = 48
      constexpr uint32_t idesc_pv = tc::instr_desc_e4m3(kD, 3 * kN) | (1u << 10) | (1u << 15) | (1u << 16);
      const uint32_t p_addr0 = smem_addr(p_buf);
      int q_valid = 0, p_valid = 0;  // valid tiles that got their QK / PV
      int prev_v = -1, prev_nv = 0;  // the held tile: its V fill (= tile index), its valid rows
      bool ok = true;
      auto wait = [&](uint64_t* bar, uint32_t parity) {
        if (ok && !mbar_wait(bar, parity)) {
          ok = false;
          *abort_flag = 1;
          set_status(a.status, PKV_DEV_TIMEOUT);
        }
        return ok;
      };
      // O += Vᵀ·P of the held tile (its P in buffer p_valid & 1)
      auto issue_pv = [&]() {
        const int b = p_valid & 1;
        const int vs = prev_v % kVStages;
        if (!wait(&v_full[vs], (prev_v / kVStages) & 1)) return;
        if (!wait(&p_full[b], (p_valid >> 1) & 1)) return;
        tc::tc_fence_after();
        const int rf = restart_flag[b];
        const bool restart = rf & 1;
        const uint32_t o_col = kColO + ((rf >> 1) & 1) * kOStride;
        const uint32_t v_addr = smem_addr(v_ring + vs * kTile8);
        const uint32_t p_addr = p_addr0 + b * kPBytes;
        const int kt = (prev_nv + 31) / 32;
        for (int kk = 0; kk < kt; ++kk) {
          // V: 32 tokens = 4 swizzle atoms of 8 rows; P: 4 groups of 8 tokens x 16 bytes, terms 2 KiB apart
          tc::umma_f8(tmem + o_col, tc::smem_desc_sw128(v_addr + kk * 4096, kTile * kRow8, 1024),
                      tc::smem_desc_plain(p_addr + kk * 512, 128, kPTerm), idesc_pv, kk > 0 || !restart);
        }
        tc::umma_commit(&o_bar[b]);
        tc::umma_commit(&v_empty[vs]);
        ++p_valid;
        prev_v = -1;
      };
      for (int n = 0; ok; ++n) {
        const int slot = n % kKStages;
        if (!wait(&k_full[slot], (n / kKStages) & 1)) break;
        const int4 mt = meta[slot];
        if (mt.w & kMetaEnd) break;
        const int nv = mt.w & 0xff;
        if (nv == 0) {
          if (prev_v >= 0) issue_pv();
          // a tile with no rows: no S to wait for, and its V fill carries no data; release both
          mbar_arrive(&k_empty[slot]);
          if (!wait(&v_full[n % kVStages], (n / kVStages) & 1)) break;
          mbar_arrive(&v_empty[n % kVStages]);
          continue;
        }
        // S = K·[hi; lo]ᵀ of tile n
        const int qs = (mt.y >> 16) & 0xf;
        const int b = q_valid & 1;
        if (q_valid >= 2 && !wait(&s_free[b], ((q_valid >> 1) - 1) & 1)) break;
        tc::tc_fence_after();
        const uint32_t k_addr = smem_addr(k_ring + slot * kTile8);
        const uint32_t q_addr = smem_addr(q_ring + qs * kQSlot);
#pragma unroll
        for (int kk = 0; kk < kD / 32; ++kk)
          tc::umma_f8(tmem + b * 32, tc::smem_desc_sw128(k_addr + kk * 32, 16, 1024),
                      tc::smem_desc_sw128(q_addr + kk * 32, 16, 1024), idesc_qk, kk > 0);
        tc::umma_commit(&s_full[b]);
        tc::umma_commit(&k_empty[slot]);  // K is free once S is done
        ++q_valid;
        // then O += Vᵀ·P of the previous valid tile
        if (prev_v >= 0) issue_pv();
        prev_v = n;
        prev_nv = nv;
      }
      if (ok && prev_v >= 0) issue_pv();
      // every MMA of this CTA is done before the tensor memory is freed
      tc::umma_commit(drain);
      mbar_wait(drain, 0);
    }
    __syncwarp();
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kRegsSoftmax));
    // ================= softmax: thread = token row of the tile = TMEM lane =================
    // With two groups, group G (warps 4G .. 4G+3) takes head pairs G, G+2, G+4, ..: local
    // head j is head 4 (j / 2) + 2G + j % 2, and both groups walk every tile together.  One
    // group takes every head (local head j = head j).
    constexpr int NL = NH / GROUPS;          // heads of one group
    constexpr int kColLanes = 32 / NL;       // lanes sharing one column after warp_col
    const int G = warp >> 2;
    const int t = tid & 127;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    float* red_max = red + G * 192;          // [4 warps][16]
    float* red_sums = red_max + 64;          // [item parity][4 warps][16]
    auto head = [&](int j) { return GROUPS == 2 ? 4 * (j >> 1) + 2 * G + (j & 1) : j; };
    float m_used[NL], lp[NL], o_reg[NL], hscale[NL];
#pragma unroll
    for (int j = 0; j < NL; ++j) m_used[j] = -INFINITY, lp[j] = 0.f, o_reg[j] = 0.f, hscale[j] = 0.f;
    float out_scale = 1.f;
    bool restart = true;
    bool pv_since_restart = false;
    int n_valid_tiles = 0;
    int obuf = 1;  // O buffer of the current item (alternates per item)
    // An item's output is written one tile later, after the next tile's P is released,
    // so its last P·V completes meanwhile instead of being waited for.
    bool fin = false;
    int4 f_mt = make_int4(0, 0, 0, 0);
    float f_o[NL], f_lp[NL], f_m[NL];
    float f_scale = 1.f;
    int f_ob = 0, f_b = 0;
    bool f_has_o = false;
    uint32_t ob_next = 0, ob_pending = 0;
    auto wait_ob = [&](int b) -> bool {
      if (!((ob_pending >> b) & 1)) return true;
      ob_pending &= ~(1u << b);
      return mbar_wait(&o_bar[b], ((ob_next >> b) & 1) ^ 1u);
    };
    // this group's heads of O buffer ob (sum of the three terms' columns) in this thread's row
    auto load_o = [&](float (&o)[NL], int ob) {
      float o3[3 * kN];
      tc::tmem_load32f_nowait(tmem + lane_base + kColO + ob * kOStride, o3);
      tc::tmem_load32f_nowait(tmem + lane_base + kColO + ob * kOStride + 32, o3 + 32);
      tc::tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < NL; ++j) {
        // register indices stay compile-time: group 1's heads are group 0's plus 2
        const int h0 = GROUPS == 2 ? 4 * (j >> 1) + (j & 1) : j;
        o[j] = G ? o3[h0 + 2] + o3[kN + h0 + 2] + o3[2 * kN + h0 + 2] : o3[h0] + o3[kN + h0] + o3[2 * kN + h0];
      }
    };
    // ---- the held item's output: O = registers + TMEM, times the V scale; denominators
    auto finalize = [&]() {
      fin = false;
      bool ok = true;
      float ot[NL];
      if (f_has_o) {
        ok = wait_ob(f_b);  // its last P·V (the latest on P buffer f_b)
        tc::tc_fence_after();
        float o[NL];
        load_o(o, f_ob);
        tc::tc_fence_before();
#pragma unroll
        for (int j = 0; j < NL; ++j) ot[j] = (f_o[j] + o[j]) * f_scale;
      } else {
#pragma unroll
        for (int j = 0; j < NL; ++j) ot[j] = f_o[j] * f_scale;
      }
      if (!ok) *abort_flag = 1;
      float* red_sum = red_sums + f_ob * 64;  // consecutive items use different halves
      const float wsum = tc::warp_col<false, NL>(f_lp, lane);
      if (lane % kColLanes == 0) red_sum[(warp & 3) * 16 + lane / kColLanes] = wsum;
      tc::named_barrier_sync(2 + G, 128);
      const int seq = f_mt.x, kvh = f_mt.y & 0xffff, part = f_mt.z & 0xffff, nparts = f_mt.z >> 16;
      const int d = t;
      const int64_t unit0 = static_cast<int64_t>(seq) * a.num_heads + kvh * g;
#pragma unroll
      for (int j = 0; j < NL; ++j) {
        const int h = head(j);
        if (h >= g) break;  // heads of a group increase with j
        const float l = red_sum[j] + red_sum[16 + j] + red_sum[32 + j] + red_sum[48 + j];
        if (nparts == 1 && !a.always_partial) {
          store_out<OUT_F32>(a, (unit0 + h) * kD + d, l > 0.f ? ot[j] / l : 0.f);
        } else {
          // unnormalised partial; the weights are held times 2^7 in both o and l, so the
          // partial's maximum is recorded as the held one minus 7 (o and l are then the sums
          // of 2^(x - m) (v, 1), as every partial a merge combines)
          const int64_t pidx = (unit0 + h) * a.max_parts + part;
          a.part_o[pidx * kD + d] = ot[j];
          if (d == 0) a.part_ml[pidx] = make_float2(f_m[j] - kPShift, l);
        }
      }
    };
    bool ended = false;
    for (int n = 0;; ++n) {
      const int slot = n % kKStages;
      bool bad = !mbar_wait(&k_full[slot], (n / kKStages) & 1);
      const int4 mt = meta[slot];
      const float2 sc = mscale[slot];
      if (bad) *abort_flag = 1;
      if (bad) break;
      if (mt.w & kMetaEnd) {
        ended = true;
        break;
      }
      const int n_valid = mt.w & 0xff;
      const uint32_t mask = (mt.w >> 8) & 0xff;
      const bool first = mt.w & kMetaFirst, last = mt.w & kMetaLast;
      if (first) {
#pragma unroll
        for (int j = 0; j < NL; ++j) m_used[j] = -INFINITY, lp[j] = 0.f, o_reg[j] = 0.f;
        restart = true;
        pv_since_restart = false;
        out_scale = sc.y;
        obuf ^= 1;
        if (n_valid > 0) {
          const int qs = (mt.y >> 16) & 0xf;  // its split queries and head scales landed with this tile
          const float base = a.scale_log2 * sc.x;
#pragma unroll
          for (int j = 0; j < NL; ++j) hscale[j] = base * qinv[qs * 16 + head(j)];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&k_empty[slot]);  // metadata (and this item's query scales) read
      if (n_valid > 0) {
        const int b = n_valid_tiles & 1;
        unsigned char* p_tile = p_buf + b * kPBytes;
        bad |= !mbar_wait(&s_full[b], (n_valid_tiles >> 1) & 1);
        tc::tc_fence_after();
        float s[2 * kN];
        tc::tmem_load32f_nowait(tmem + lane_base + b * 32, s);
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[b]);
        bad |= !wait_ob(b);  // P buffer b: the P·V of two valid tiles back is done
        const bool valid = t < n_valid && ((mask >> (t / kChunk)) & 1);
        if (n_valid < kTile || mask != 0xffu) {  // uniform: the tile has rows outside the context
          // V rows outside the context may hold anything (even NaN codes): zero them once the
          // tile's V has landed (each group half of the row)
          const int vs = n % kVStages;
          bad |= !mbar_wait(&v_full[vs], (n / kVStages) & 1);
          if (!valid) {
            uint4* vr = reinterpret_cast<uint4*>(v_ring + vs * kTile8 + t * kRow8) + (8 / GROUPS) * G;
#pragma unroll
            for (int c = 0; c < 8 / GROUPS; ++c) vr[c] = make_uint4(0, 0, 0, 0);
          }
        }
        float x[NL];
        bool need = false;
#pragma unroll
        for (int j = 0; j < NL; ++j) {
          const int h0 = GROUPS == 2 ? 4 * (j >> 1) + (j & 1) : j;  // compile-time register indices
          const float sv = G ? s[h0 + 2] + s[kN + h0 + 2] : s[h0] + s[kN + h0];
          x[j] = (valid && head(j) < g) ? sv * hscale[j] : -INFINITY;
          need |= x[j] > m_used[j] + kRescaleLog2;
        }
        // P of this token: head pair (2k, 2k+1) of each term is 2 bytes at 2k of the
        // term's 16-byte chunk at (t/8)*128 + (t%8)*16 of its 2 KiB third of the buffer.
        float pv[NL];
        auto write_p = [&]() {
          // global head pair of local pair k: 2k + G with two groups, k with one (2 bytes per pair)
          unsigned char* row = p_tile + (t >> 3) * 128 + (t & 7) * 16 + (GROUPS == 2 ? 2 * G : 0);
#pragma unroll
          for (int k = 0; k < NL / 2; ++k) {
            const int j0 = 2 * k, j1 = 2 * k + 1;
            const float p0 = (valid && head(j0) < g && m_used[j0] > -INFINITY)
                                 ? fast_exp2(x[j0] - m_used[j0] + kPShift) : 0.f;
            const float p1 = (valid && head(j1) < g && m_used[j1] > -INFINITY)
                                 ? fast_exp2(x[j1] - m_used[j1] + kPShift) : 0.f;
            uint32_t ph, pm, pl, sum;
            split_p2(pack_f16x2(p0, p1), ph, pm, pl, sum);
            pv[j0] = f16lo(sum);
            pv[j1] = f16hi(sum);
            // the codes are the top bytes of the two f16 halves
            const int pk = GROUPS == 2 ? 4 * k : 2 * k;
            *reinterpret_cast<uint16_t*>(row + pk) = static_cast<uint16_t>(__byte_perm(ph, 0, 0x0031));
            *reinterpret_cast<uint16_t*>(row + kPTerm + pk) = static_cast<uint16_t>(__byte_perm(pm, 0, 0x0031));
            *reinterpret_cast<uint16_t*>(row + 2 * kPTerm + pk) = static_cast<uint16_t>(__byte_perm(pl, 0, 0x0031));
          }
        };
        if (bad) *abort_flag = 1;
        bool need_any = true;  // an item's first tile always sets the held maximum
        if (!first) {
          write_p();
          if (tid == 0) restart_flag[b] = (restart ? 1 : 0) | (obuf << 1);
          fence_proxy_async_smem();
          // one decision for both groups: a rescale restarts the shared O
          need_any = tc::named_barrier_or(1, kSoftmax, need || bad);
          if (*abort_flag) break;
        }
        if (need_any) {
          // a score outgrew the held maximum (or none is held yet): take the tile
          // maximum, fold the accumulated P·V into registers at the old scale, rewrite P
          const float wmax = tc::warp_col<true, NL>(x, lane);
          if (lane % kColLanes == 0) red_max[(warp & 3) * 16 + lane / kColLanes] = wmax;
          bool ok = true;
          if (pv_since_restart) {  // this item's O is folded below: its P·Vs must be complete
            ok = wait_ob(0);
            ok &= wait_ob(1);
          }
          if (!ok) *abort_flag = 1;
          // both groups: every P·V into the shared O is complete before either folds it
          tc::named_barrier_sync(1, kSoftmax);
          if (*abort_flag) break;
          float alpha[NL];
#pragma unroll
          for (int j = 0; j < NL; ++j) {
            const float tmax = fmaxf(fmaxf(red_max[j], red_max[16 + j]), fmaxf(red_max[32 + j], red_max[48 + j]));
            if (head(j) < g) {
              const float m_new = fmaxf(m_used[j], tmax);
              alpha[j] = m_used[j] == -INFINITY ? 0.f : fast_exp2(m_used[j] - m_new);
              m_used[j] = m_new;
            } else {
              alpha[j] = 1.f;
            }
          }
          tc::tc_fence_after();
          if (pv_since_restart) {
            float o[NL];
            load_o(o, obuf);
#pragma unroll
            for (int j = 0; j < NL; ++j) o_reg[j] = (o_reg[j] + o[j]) * alpha[j];
          } else {
#pragma unroll
            for (int j = 0; j < NL; ++j) o_reg[j] *= alpha[j];
          }
          tc::tc_fence_before();
#pragma unroll
          for (int j = 0; j < NL; ++j) lp[j] *= alpha[j];
          restart = true;
          pv_since_restart = false;
          write_p();
          if (tid == 0) restart_flag[b] = 1 | (obuf << 1);
          fence_proxy_async_smem();
          tc::named_barrier_sync(2 + G, 128);  // the group's maxima read before they are rewritten
        }
#pragma unroll
        for (int j = 0; j < NL; ++j)
          if (head(j) < g) lp[j] += pv[j];
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
        for (int j = 0; j < NL; ++j) f_o[j] = o_reg[j], f_lp[j] = lp[j], f_m[j] = m_used[j];
        f_scale = out_scale;
        f_ob = obuf;
        f_has_o = pv_since_restart;
        f_b = (n_valid_tiles - 1) & 1;  // P buffer of the item's last valid tile
      }
    }
    if (ended && fin) finalize();
    if (*abort_flag && tid == 0) set_status(a.status, PKV_DEV_TIMEOUT);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

// ---- query split ------------------------------------------------------------------
//
// Once per call, before the main kernel: every (sequence, kv head) unit's g query heads as
// e4m3 [hi; lo] rows, one warp per unit.  Lane l takes head r = l / 2, half h = l % 2 (dims
// 64h .. 64h+63).  The head's largest |q| is brought into [128, 256) by a power of two 2^e;
// hi is q·2^e rounded to e4m3, lo the remainder rounded to e4m3.  Row r holds hi of head r,
// row 16 + r its lo, 128 codes each (plain rows: the main kernel's tensor map applies the
// 128-byte swizzle on load); rows of heads g .. 15 are zero.  2^-e goes to q_inv[unit][r].
constexpr int kSplitWarps = 4;

// One (sequence, kv head): its g query rows split into e4m3 [hi; lo] rows and a power-of-two
// scale per head (lane = row r, half h).
__device__ __forceinline__ void split_unit(const DecodeArgs& a, int64_t unit, int lane) {
  const int seq = static_cast<int>(unit / a.num_kv_heads), kvh = static_cast<int>(unit % a.num_kv_heads);
  const int g = a.group;
  const int r = lane >> 1, h = lane & 1;
  const bool live = r < g;
  const uint4* src = reinterpret_cast<const uint4*>(a.query + (static_cast<int64_t>(seq) * a.num_heads + kvh * g +
                                                               (live ? r : 0)) * kD + 64 * h);
  uint4 v[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) v[c] = live ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
  float m = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) m = fmaxf(m, fmaxf(fabsf(bf16lo(w[i])), fabsf(bf16hi(w[i]))));
  }
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  const int E = static_cast<int>((__float_as_uint(m) >> 23) & 0xff);
  const int e = E == 0 ? 0 : min(134 - E, 126);
  const float up = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
  uint8_t* dst = a.q_split + unit * static_cast<int64_t>(kQSplitUnitBytes);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 x0 = v[2 * j], x1 = v[2 * j + 1];  // dims 64h + 16j + 0..7, + 8..15
    const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    uint32_t q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = split_q2(bf16lo(w[i]) * up, bf16hi(w[i]) * up);
    const uint4 hi4 = make_uint4(__byte_perm(q[0], q[1], 0x5410), __byte_perm(q[2], q[3], 0x5410),
                                 __byte_perm(q[4], q[5], 0x5410), __byte_perm(q[6], q[7], 0x5410));
    const uint4 lo4 = make_uint4(__byte_perm(q[0], q[1], 0x7632), __byte_perm(q[2], q[3], 0x7632),
                                 __byte_perm(q[4], q[5], 0x7632), __byte_perm(q[6], q[7], 0x7632));
    *reinterpret_cast<uint4*>(dst + r * 128 + (4 * h + j) * 16) = hi4;
    *reinterpret_cast<uint4*>(dst + (16 + r) * 128 + (4 * h + j) * 16) = lo4;
  }
  if (h == 0) a.q_inv[unit * 16 + r] = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
}

__global__ void __launch_bounds__(kSplitWarps * 32) split_queries_kernel(const DecodeArgs a) {
  griddep_launch_dependents();  // the decode kernel may be scheduled now
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t unit = static_cast<int64_t>(blockIdx.x) * kSplitWarps + warp;
  // The split reads only the caller's queries and writes only its own rows, so it runs beside
  // the plan kernel before it; it waits for the plan only to end after it.
  if (unit < static_cast<int64_t>(a.num_seqs) * a.num_kv_heads) split_unit(a, unit, lane);  // warp-uniform
  griddep_wait();
}

// ---- host side -----------------------------------------------------------------

// 2-D view [rows, 128] bytes with a 128-byte swizzle, box 128 x box_rows: the e4m3 pool
// (16-row slices) or the split queries (32 rows per unit).
static int encode_map(CUtensorMap* map, const void* base, uint64_t rows, int box_rows, const char* what) {
  auto encode = tc::tensor_map_encoder();
  if (!encode) return set_error(PKV_ERR_CUDA, "decode (8-bit tensor): cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), rows};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD)};
  cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                      const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(PKV_ERR_CUDA, "decode (8-bit tensor): tensor map for %s failed (%d)", what, (int)r);
  return PKV_OK;
}

template <bool OUT_F32, int NH>
static int launch(const Args& args, cudaStream_t stream) {
  constexpr int GROUPS = NH <= PKV_FP8_ONE_GROUP_MAX_NH ? 1 : 2;
  using C = Cfg<GROUPS>;
  constexpr int kSmemBytes = C::kSmemBytes;
  auto kernel = decode_gqa_tc_fp8_kernel<OUT_F32, NH, GROUPS>;
  static PerDevice<int> setup;
  int dev = 0, sms = 0;
  const int st = set_smem_limit_once(setup, kernel, kSmemBytes, &dev);
  if (st != 0)
    return set_error(PKV_ERR_CUDA, "decode (8-bit tensor) setup: %s", cudaGetErrorString(static_cast<cudaError_t>(st)));
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaError_t e =
      launch_after_previous(kernel, dim3(std::max(1, sms * C::kCtasPerSm)), dim3(C::kThreads), kSmemBytes, stream, args);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(PKV_ERR_CUDA, "decode (8-bit tensor) launch: %s", cudaGetErrorString(e));
  return PKV_OK;
}

}  // namespace tc8

int launch_decode_tensor_fp8(const DecodeArgs& a, int head_dim, bool out_f32, cudaStream_t stream) {
  if (!tensor_path_supports(a.group, head_dim))
    return set_error(PKV_ERR_UNSUPPORTED, "decode (8-bit tensor): group %d / head_dim %d not supported", a.group,
                     head_dim);
  tc8::Args args;
  args.a = a;
  const uint64_t pool_rows = static_cast<uint64_t>(a.num_blocks) * a.num_kv_heads * a.block_size;
  if (!a.q_split || !a.q_inv) return set_error(PKV_ERR_INVALID, "decode (8-bit tensor): no split-query workspace");
  const uint64_t units = static_cast<uint64_t>(a.num_seqs) * a.num_kv_heads;
  const int rows = tc8::box_rows(a.block_size);
  int rc = tc8::encode_map(&args.tm_k, a.key_cache8, pool_rows, rows, "key_cache");
  if (rc == PKV_OK) rc = tc8::encode_map(&args.tm_v, a.value_cache8, pool_rows, rows, "value_cache");
  if (rc == PKV_OK) rc = tc8::encode_map(&args.tm_q, a.q_split, units * 32, 32, "split queries");
  if (rc != PKV_OK) return rc;
  if (units > 0) {
    const unsigned grid = static_cast<unsigned>((units + tc8::kSplitWarps - 1) / tc8::kSplitWarps);
    cudaError_t e = launch_after_previous(tc8::split_queries_kernel, dim3(grid), dim3(tc8::kSplitWarps * 32), 0,
                                          stream, a);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess)
      return set_error(PKV_ERR_CUDA, "decode (8-bit tensor) query split launch: %s", cudaGetErrorString(e));
  }
  if (a.group <= 4)
    rc = out_f32 ? tc8::launch<true, 4>(args, stream) : tc8::launch<false, 4>(args, stream);
  else if (a.group <= 8)
    rc = out_f32 ? tc8::launch<true, 8>(args, stream) : tc8::launch<false, 8>(args, stream);
  else
    rc = out_f32 ? tc8::launch<true, 16>(args, stream) : tc8::launch<false, 16>(args, stream);
  if (rc != PKV_OK) return rc;
  return a.always_partial ? PKV_OK : launch_merge_partials(a, out_f32, stream);
}

}  // namespace pkv
