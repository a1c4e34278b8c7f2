// Host planner of the shared-prefix decode (pkv_shared_plan).
//
// Blocks that several tables hold at the same positions (a system prompt shared by
// many requests, the prompt and generated text a parent shares with its beams; Outcome
// School explainer, "内存共享") hold the same keys and values for all of those rows.
// The plan finds, among ADJACENT rows of the batch, maximal runs of such blocks and
// lays out the work of the shared-prefix decode (its header comment in pkv.h gives the
// arithmetic): segments cut into key chunks ("parts"), the pairs of 128-row query tiles
// of every part, each row's private remainder, and the list of partial results each
// row merges.
//
// Segments form a tree over row ranges.  At table position k, a range of rows that
// already shares positions [0, k) splits into maximal runs of consecutive rows whose
// block at k is the same and full for all of them (a block is full for a row when all
// block_size of its tokens are below the row's length).  A run of at least min_rows
// rows extends its segment over every following position where the same holds, and
// is then split again at the first position where it does not.  Every row's segments
// are therefore a chain covering its positions [0, k_r); the rest is private.
#include <algorithm>
#include <cstring>
#include <vector>

#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr int kTileRows = 128;       // query rows of one tile of the shared phase (MMA M)
// Shared-phase work items the automatic key chunk aims for: the phase runs beside the private
// decode, so it needs no full wave of its own, and longer chunks leave fewer partials to merge.
constexpr int kItemsTarget = 64;

struct Segment {
  int row0, nrows, block0, nblocks;
};

struct Part {
  int seg, key0, nkeys;  // keys from the segment's first token
};

inline size_t align16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" int pkv_shared_plan(const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                               int num_seqs, int num_heads, int num_kv_heads, int block_size, int min_rows,
                               int key_chunk, void* plan, size_t plan_bytes, pkv_shared_plan_info* info) {
  clear_error();
  if (!info) return set_error(PKV_ERR_INVALID, "shared_plan: null info");
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || num_heads <= 0 || num_kv_heads <= 0 || block_size <= 0 ||
      min_rows < 2 || key_chunk < 0 || key_chunk % 128 != 0)
    return set_error(PKV_ERR_INVALID, "shared_plan: bad sizes");
  if (num_heads % num_kv_heads != 0 || kTileRows % (num_heads / num_kv_heads) != 0)
    return set_error(PKV_ERR_UNSUPPORTED, "shared_plan: num_heads / num_kv_heads must divide 128");
  if (num_seqs > 0 && (!block_tables || !context_lens)) return set_error(PKV_ERR_INVALID, "shared_plan: null pointer");
  const int group = num_heads / num_kv_heads;
  const int max_tokens = max_blocks_per_seq * block_size;
  for (int r = 0; r < num_seqs; ++r)
    if (context_lens[r] < 0 || context_lens[r] > max_tokens)
      return set_error(PKV_ERR_INVALID, "shared_plan: context_lens[%d] = %d outside [0, %d]", r, context_lens[r],
                       max_tokens);

  auto full = [&](int r, int k) { return k < max_blocks_per_seq && (k + 1) * block_size <= context_lens[r]; };
  auto at = [&](int r, int k) { return block_tables[static_cast<int64_t>(r) * max_blocks_per_seq + k]; };

  // ---- segments: a work list of (row range, position) that already share [0, position)
  std::vector<Segment> segs;
  std::vector<int> depth(num_seqs, 0);  // block offset where each row's private part starts
  struct Range {
    int r0, r1, k;
  };
  std::vector<Range> work;
  if (num_seqs > 0) work.push_back({0, num_seqs, 0});
  while (!work.empty()) {
    const Range w = work.back();
    work.pop_back();
    int r = w.r0;
    while (r < w.r1) {
      if (!full(r, w.k)) {
        ++r;
        continue;
      }
      int s = r + 1;
      while (s < w.r1 && full(s, w.k) && at(s, w.k) == at(r, w.k)) ++s;
      if (s - r >= min_rows) {
        // k2: the first position past w.k where some row of r..s-1 has no full block or a
        // block other than row r's (each row's table scanned along its own memory)
        int k2 = max_blocks_per_seq;
        const int32_t* base = block_tables + static_cast<int64_t>(r) * max_blocks_per_seq;
        for (int q = r; q < s; ++q) {
          const int32_t* row = block_tables + static_cast<int64_t>(q) * max_blocks_per_seq;
          const int lim = std::min(k2, std::min(context_lens[q] / block_size, max_blocks_per_seq));
          int k = w.k + 1;
          while (k < lim && row[k] == base[k]) ++k;
          k2 = k;
        }
        segs.push_back({r, s - r, w.k, k2 - w.k});
        for (int q = r; q < s; ++q) depth[q] = k2;
        work.push_back({r, s, k2});
      }
      r = s;
    }
  }
  // Deterministic order: by first row, then position (parents before children).
  std::sort(segs.begin(), segs.end(), [](const Segment& a, const Segment& b) {
    return a.row0 != b.row0 ? a.row0 < b.row0 : a.block0 < b.block0;
  });

  // ---- parts: each segment cut into key chunks
  const int tile_rows = kTileRows / group;  // batch rows per query tile
  const int pair_rows = 2 * tile_rows;
  auto count_items = [&](int chunk) {
    int64_t items = 0;
    for (const Segment& sg : segs) {
      const int64_t nk = static_cast<int64_t>(sg.nblocks) * block_size;
      items += ((nk + chunk - 1) / chunk) * ((sg.nrows + pair_rows - 1) / pair_rows);
    }
    return items * num_kv_heads;
  };
  int chunk = key_chunk;
  if (chunk == 0) {
    chunk = 2048;
    while (chunk > 128 && count_items(chunk) < kItemsTarget) chunk /= 2;
  }
  std::vector<Part> parts;
  for (int i = 0; i < static_cast<int>(segs.size()); ++i) {
    const int nk = segs[i].nblocks * block_size;
    for (int k0 = 0; k0 < nk; k0 += chunk) parts.push_back({i, k0, std::min(chunk, nk - k0)});
  }
  // Parts with more keys first (load balance); a part's tile pairs stay adjacent.
  std::stable_sort(parts.begin(), parts.end(), [](const Part& a, const Part& b) { return a.nkeys > b.nkeys; });

  int64_t n_entries = 0, n_partials = 0, shared_tokens = 0, shared_row_tokens = 0;
  for (const Part& p : parts) {
    const Segment& sg = segs[p.seg];
    n_entries += (sg.nrows + pair_rows - 1) / pair_rows;
    n_partials += sg.nrows;
  }
  for (const Segment& sg : segs) {
    shared_tokens += static_cast<int64_t>(sg.nblocks) * block_size;
    shared_row_tokens += static_cast<int64_t>(sg.nblocks) * block_size * sg.nrows;
  }
  if (n_entries > (1 << 30) || n_partials > (1 << 30))
    return set_error(PKV_ERR_INVALID, "shared_plan: plan too large");
  int max_suffix = 0;
  for (int r = 0; r < num_seqs; ++r) max_suffix = std::max(max_suffix, context_lens[r] - depth[r] * block_size);

  pkv_shared_plan_info in{};
  in.num_seqs = num_seqs;
  in.num_segments = static_cast<int32_t>(segs.size());
  in.num_parts = static_cast<int32_t>(parts.size());
  in.num_entries = static_cast<int32_t>(n_entries);
  in.num_partials = static_cast<int32_t>(n_partials);
  in.max_suffix_len = max_suffix;
  in.key_chunk = chunk;
  in.group = group;
  in.block_size = block_size;
  in.max_blocks_per_seq = max_blocks_per_seq;
  in.shared_row_tokens = shared_row_tokens;
  in.shared_tokens = shared_tokens;
  size_t off = 0;
  in.off_entries = off;
  off = align16(off + static_cast<size_t>(n_entries) * 16);
  in.off_parts = off;
  off = align16(off + parts.size() * 32);
  in.off_suffix_lens = off;
  off = align16(off + static_cast<size_t>(num_seqs) * 4);
  in.off_block_offset = off;
  off = align16(off + static_cast<size_t>(num_seqs) * 4);
  in.off_row_start = off;
  off = align16(off + static_cast<size_t>(num_seqs + 1) * 4);
  in.off_row_ids = off;
  off = align16(off + static_cast<size_t>(n_partials) * 4);
  in.bytes = std::max<size_t>(off, 16);
  *info = in;
  if (!plan) return PKV_OK;
  if (plan_bytes < in.bytes)
    return set_error(PKV_ERR_INVALID, "shared_plan: plan buffer of %zu bytes, %zu needed", plan_bytes,
                     static_cast<size_t>(in.bytes));

  unsigned char* base = static_cast<unsigned char*>(plan);
  std::memset(base, 0, in.bytes);
  int32_t* entries = reinterpret_cast<int32_t*>(base + in.off_entries);
  int32_t* pdesc = reinterpret_cast<int32_t*>(base + in.off_parts);
  int32_t* suffix_lens = reinterpret_cast<int32_t*>(base + in.off_suffix_lens);
  int32_t* block_offset = reinterpret_cast<int32_t*>(base + in.off_block_offset);
  int32_t* row_start = reinterpret_cast<int32_t*>(base + in.off_row_start);
  int32_t* row_ids = reinterpret_cast<int32_t*>(base + in.off_row_ids);

  // partial ids: part i covers rows row0 .. row0 + nrows - 1 with ids first .. first + nrows - 1;
  // its blocks take the scratch blocks base .. base + keys / block_size - 1 (the 8-bit run
  // widens every part's blocks into a scratch pool in this order)
  std::vector<int> first(parts.size());
  std::vector<int> per_row(num_seqs + 1, 0);
  int next_id = 0, e = 0, next_block = 0;
  for (size_t i = 0; i < parts.size(); ++i) {
    const Segment& sg = segs[parts[i].seg];
    first[i] = next_id;
    next_id += sg.nrows;
    int32_t* d = pdesc + 8 * i;
    d[0] = sg.row0;                                      // table row holding the segment's blocks
    d[1] = sg.block0 + parts[i].key0 / block_size;       // its first block (table position)
    d[2] = parts[i].nkeys;
    d[3] = sg.row0;
    d[4] = sg.nrows;
    d[5] = first[i];
    d[6] = next_block;
    next_block += parts[i].nkeys / block_size;
    for (int r0 = 0; r0 < sg.nrows; r0 += pair_rows, ++e) {
      const int na = std::min(tile_rows, sg.nrows - r0);
      const int nb = std::max(0, std::min(tile_rows, sg.nrows - r0 - tile_rows));
      int32_t* en = entries + 4 * e;
      en[0] = sg.row0 + r0;
      en[1] = 0;
      en[2] = na | (nb << 8);
      en[3] = static_cast<int32_t>(i);
    }
    for (int q = sg.row0; q < sg.row0 + sg.nrows; ++q) ++per_row[q + 1];
  }
  for (int r = 0; r < num_seqs; ++r) per_row[r + 1] += per_row[r];
  std::vector<int> fill(per_row.begin(), per_row.end() - 1);
  for (size_t i = 0; i < parts.size(); ++i) {
    const Segment& sg = segs[parts[i].seg];
    for (int q = 0; q < sg.nrows; ++q) row_ids[fill[sg.row0 + q]++] = first[i] + q;
  }
  for (int r = 0; r <= num_seqs; ++r) row_start[r] = per_row[r];
  for (int r = 0; r < num_seqs; ++r) {
    block_offset[r] = depth[r];
    suffix_lens[r] = context_lens[r] - depth[r] * block_size;
  }
  return PKV_OK;
}
