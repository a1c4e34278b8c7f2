// Host block manager: FIFO free list, per-block reference counts and per-sequence
// block tables.
//
// Outcome School vLLM explainer, "vLLM的核心创新：PagedAttention": blocks are taken
// only when a request needs room, need not be contiguous, are recorded in order in
// the request's block table, and all go back to the shared pool when it finishes;
// "内存共享": identical prefixes and beams point their tables at the same blocks.
// The copy-on-write rule for a shared, partially filled last block and the FIFO
// order of the free list are this library's readings (documented in pkv.h).
//
// Swap space (intelliparadigm article §4.2 OOM错误: swap_space extends the pool into
// host memory): a second pool of host blocks; swap_out / swap_in move whole
// sequences between the pools and return the block pairs to copy.
// Automatic prefix caching ("内存共享": identical prefixes keep one copy): full
// prompt blocks are registered under a chain hash of their token ids; a later prompt
// takes its longest registered leading run.  A registered block with no references
// stays registered in the free list until the list hands it out again.
#include <algorithm>
#include <cstring>
#include <deque>
#include <new>
#include <unordered_map>
#include <utility>
#include <vector>

#include "pkv_internal.h"

using pkv::set_error;

namespace {

// FIFO of free block ids with O(1) removal from the middle (a cached block taken
// back), as a doubly linked list threaded through two arrays.
struct FreeList {
  std::vector<int32_t> next, prev;
  std::vector<char> in;
  int32_t head = -1, tail = -1;
  int count = 0;
  void init(int n) {
    next.assign(n, -1);
    prev.assign(n, -1);
    in.assign(n, 0);
  }
  bool empty() const { return count == 0; }
  int size() const { return count; }
  void push_back(int32_t b) {
    next[b] = -1;
    prev[b] = tail;
    if (tail >= 0) next[tail] = b; else head = b;
    tail = b;
    in[b] = 1;
    ++count;
  }
  void remove(int32_t b) {
    if (prev[b] >= 0) next[prev[b]] = next[b]; else head = next[b];
    if (next[b] >= 0) prev[next[b]] = prev[b]; else tail = prev[b];
    in[b] = 0;
    --count;
  }
  int32_t pop_front() {
    const int32_t b = head;
    remove(b);
    return b;
  }
};

constexpr uint64_t kFnvOffset = 0xcbf29ce484222325ull;
constexpr uint64_t kFnvPrime = 0x100000001b3ull;

// FNV-1a-64 of the parent hash (8 bytes, little-endian) followed by the block's
// token ids (4 bytes each, little-endian).
uint64_t block_hash(uint64_t parent, const int32_t* tokens, int n) {
  uint64_t h = kFnvOffset;
  for (int i = 0; i < 8; ++i) {
    h ^= (parent >> (8 * i)) & 0xffu;
    h *= kFnvPrime;
  }
  for (int t = 0; t < n; ++t) {
    const uint32_t v = static_cast<uint32_t>(tokens[t]);
    for (int i = 0; i < 4; ++i) {
      h ^= (v >> (8 * i)) & 0xffu;
      h *= kFnvPrime;
    }
  }
  return h;
}

}  // namespace

struct pkv_bm {
  struct Seq {
    std::vector<int32_t> table;  // device blocks, or host blocks while swapped out
    int len = 0;
    bool swapped = false;
    // Token history for the prefix cache: known for sequences created from token
    // ids and kept by append_tokens; lost (false) after a plain append_slots.
    bool tracked = false;
    uint64_t parent = 0;           // chain hash of the last full block
    std::vector<int32_t> partial;  // token ids of the block being filled
    uint64_t stamp = 0;            // the last append call that listed it (repeats are rejected)
  };
  int num_blocks = 0;
  int block_size = 0;
  FreeList free_list;
  std::vector<int32_t> ref;
  std::unordered_map<int64_t, Seq> seqs;
  // swap space
  int num_host_blocks = 0;
  std::deque<int32_t> host_free;
  std::vector<int32_t> host_ref;
  // prefix cache: hash -> block, and the hash a block is registered under
  std::unordered_map<uint64_t, int32_t> cached;
  std::vector<uint64_t> block_hash_of;
  std::vector<char> registered;
  // Scratch for the dry run of append_slots: per-block pending reference change.
  std::vector<int32_t> pending;
  std::vector<int32_t> touched;
  // Scratch of append calls: the listed sequences, and the call's stamp.
  std::vector<Seq*> listed;
  uint64_t append_calls = 0;

  bool valid_block(int32_t b) const { return b >= 0 && b < num_blocks; }
  int blocks_for(int tokens) const { return (tokens + block_size - 1) / block_size; }

  int32_t take() {
    const int32_t b = free_list.pop_front();
    ref[b] = 1;
    if (registered[b]) {  // handing a cached block out evicts it
      cached.erase(block_hash_of[b]);
      registered[b] = 0;
    }
    return b;
  }
  void drop(int32_t b) {
    if (--ref[b] == 0) free_list.push_back(b);
  }
  void host_drop(int32_t b) {
    if (--host_ref[b] == 0) host_free.push_back(b);
  }
};

extern "C" pkv_bm* pkv_bm_create(int num_blocks, int block_size, const int32_t* initial_order) {
  if (num_blocks <= 0 || block_size <= 0) {
    set_error(PKV_ERR_INVALID, "pkv_bm_create: num_blocks and block_size must be positive");
    return nullptr;
  }
  pkv_bm* bm = new (std::nothrow) pkv_bm();
  if (!bm) {
    set_error(PKV_ERR_OOM, "pkv_bm_create: host allocation failed");
    return nullptr;
  }
  bm->num_blocks = num_blocks;
  bm->block_size = block_size;
  bm->ref.assign(num_blocks, 0);
  bm->pending.assign(num_blocks, 0);
  bm->free_list.init(num_blocks);
  bm->block_hash_of.assign(num_blocks, 0);
  bm->registered.assign(num_blocks, 0);
  if (initial_order) {
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
      int32_t b = initial_order[i];
      if (b < 0 || b >= num_blocks || seen[b]) {
        delete bm;
        set_error(PKV_ERR_INVALID, "pkv_bm_create: initial_order is not a permutation of 0..%d", num_blocks - 1);
        return nullptr;
      }
      seen[b] = 1;
      bm->free_list.push_back(b);
    }
  } else {
    for (int i = 0; i < num_blocks; ++i) bm->free_list.push_back(i);
  }
  return bm;
}

extern "C" void pkv_bm_destroy(pkv_bm* bm) { delete bm; }

extern "C" int pkv_bm_num_blocks(const pkv_bm* bm) { return bm ? bm->num_blocks : PKV_ERR_INVALID; }
extern "C" int pkv_bm_block_size(const pkv_bm* bm) { return bm ? bm->block_size : PKV_ERR_INVALID; }
extern "C" int pkv_bm_num_free(const pkv_bm* bm) {
  return bm ? bm->free_list.size() : PKV_ERR_INVALID;
}

extern "C" int pkv_bm_free_list(const pkv_bm* bm, int32_t* out, int cap) {
  if (!bm || (cap > 0 && !out)) return set_error(PKV_ERR_INVALID, "pkv_bm_free_list: bad arguments");
  int n = 0;
  for (int32_t b = bm->free_list.head; b >= 0 && n < cap; b = bm->free_list.next[b]) out[n++] = b;
  return n;
}

extern "C" int pkv_bm_alloc(pkv_bm* bm, int32_t* block_out) {
  if (!bm || !block_out) return set_error(PKV_ERR_INVALID, "pkv_bm_alloc: bad arguments");
  if (bm->free_list.empty()) return set_error(PKV_ERR_OOM, "pkv_bm_alloc: pool exhausted");
  *block_out = bm->take();
  return PKV_OK;
}

extern "C" int pkv_bm_incref(pkv_bm* bm, int32_t block) {
  if (!bm || !bm->valid_block(block) || bm->ref[block] <= 0)
    return set_error(PKV_ERR_INVALID, "pkv_bm_incref: block %d is not live", block);
  ++bm->ref[block];
  return PKV_OK;
}

extern "C" int pkv_bm_decref(pkv_bm* bm, int32_t block) {
  if (!bm || !bm->valid_block(block) || bm->ref[block] <= 0)
    return set_error(PKV_ERR_INVALID, "pkv_bm_decref: block %d is not live", block);
  bm->drop(block);
  return PKV_OK;
}

extern "C" int pkv_bm_refcount(const pkv_bm* bm, int32_t block) {
  if (!bm || !bm->valid_block(block)) return set_error(PKV_ERR_INVALID, "pkv_bm_refcount: bad block %d", block);
  return bm->ref[block];
}

extern "C" int pkv_bm_add_seq(pkv_bm* bm, int64_t seq_id, int num_tokens, const int32_t* shared_prefix_blocks,
                              int n_shared) {
  if (!bm || num_tokens < 0 || n_shared < 0 || (n_shared > 0 && !shared_prefix_blocks))
    return set_error(PKV_ERR_INVALID, "pkv_bm_add_seq: bad arguments");
  if (bm->seqs.count(seq_id)) return set_error(PKV_ERR_INVALID, "pkv_bm_add_seq: sequence %lld exists", (long long)seq_id);
  if (static_cast<int64_t>(n_shared) * bm->block_size > num_tokens)
    return set_error(PKV_ERR_INVALID, "pkv_bm_add_seq: shared prefix longer than the sequence");
  for (int i = 0; i < n_shared; ++i) {
    int32_t b = shared_prefix_blocks[i];
    if (!bm->valid_block(b) || bm->ref[b] <= 0)
      return set_error(PKV_ERR_INVALID, "pkv_bm_add_seq: shared block %d is not live", b);
  }
  int fresh = bm->blocks_for(num_tokens) - n_shared;
  if (fresh > bm->free_list.size())
    return set_error(PKV_ERR_OOM, "pkv_bm_add_seq: pool exhausted (%d blocks needed, %zu free)", fresh,
                     bm->free_list.size());
  pkv_bm::Seq seq;
  seq.table.reserve(n_shared + fresh);
  for (int i = 0; i < n_shared; ++i) {
    ++bm->ref[shared_prefix_blocks[i]];
    seq.table.push_back(shared_prefix_blocks[i]);
  }
  for (int i = 0; i < fresh; ++i) seq.table.push_back(bm->take());
  seq.len = num_tokens;
  bm->seqs.emplace(seq_id, std::move(seq));
  return PKV_OK;
}

extern "C" int pkv_bm_fork(pkv_bm* bm, int64_t parent, int64_t child) {
  if (!bm) return set_error(PKV_ERR_INVALID, "pkv_bm_fork: null manager");
  auto it = bm->seqs.find(parent);
  if (it == bm->seqs.end() || bm->seqs.count(child) || it->second.swapped)
    return set_error(PKV_ERR_INVALID, "pkv_bm_fork: unknown parent %lld or existing child %lld", (long long)parent,
                     (long long)child);
  pkv_bm::Seq copy = it->second;
  for (int32_t b : copy.table) ++bm->ref[b];
  bm->seqs.emplace(child, std::move(copy));
  return PKV_OK;
}

// One new position per listed sequence (all-or-nothing), then, with token ids, the
// prefix-cache bookkeeping of each tracked sequence; without them the sequences'
// token history is lost.
static int append_impl(pkv_bm* bm, const int64_t* seq_ids, const int32_t* tokens, int n, int64_t* slots_out,
                       int64_t* cow_pairs_out, int* n_cow_out) {
  if (!bm || n < 0 || (n > 0 && (!seq_ids || !slots_out || !cow_pairs_out)) || !n_cow_out)
    return set_error(PKV_ERR_INVALID, "pkv_bm_append_slots: bad arguments");
  *n_cow_out = 0;
  // Validate ids (known, distinct: a sequence already stamped by this call is a repeat) and
  // resolve them once.
  std::vector<pkv_bm::Seq*>& seqs = bm->listed;
  seqs.resize(static_cast<size_t>(n));
  const uint64_t stamp = ++bm->append_calls;
  for (int i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end() || it->second.swapped || it->second.stamp == stamp)
      return set_error(PKV_ERR_INVALID, "pkv_bm_append_slots: unknown, repeated or swapped-out sequence %lld",
                       (long long)seq_ids[i]);
    it->second.stamp = stamp;
    seqs[i] = &it->second;
  }
  // Dry run: count fresh blocks, following reference counts as earlier sequences
  // of this call give up their share of a block.
  int need = 0;
  for (int i = 0; i < n; ++i) {
    pkv_bm::Seq& s = *seqs[i];
    if (s.len % bm->block_size == 0) {
      ++need;
    } else {
      int32_t last = s.table.back();
      if (bm->ref[last] + bm->pending[last] > 1) {
        ++need;
        if (bm->pending[last] == 0) bm->touched.push_back(last);
        --bm->pending[last];
      }
    }
  }
  for (int32_t b : bm->touched) bm->pending[b] = 0;
  bm->touched.clear();
  if (need > bm->free_list.size())
    return set_error(PKV_ERR_OOM, "pkv_bm_append_slots: pool exhausted (%d blocks needed, %d free)", need,
                     bm->free_list.size());
  int n_cow = 0;
  for (int i = 0; i < n; ++i) {
    pkv_bm::Seq& s = *seqs[i];
    const int row = s.len % bm->block_size;
    if (row == 0) {
      s.table.push_back(bm->take());
    } else if (bm->ref[s.table.back()] > 1) {
      int32_t old = s.table.back();
      int32_t fresh = bm->take();
      cow_pairs_out[2 * n_cow] = old;
      cow_pairs_out[2 * n_cow + 1] = fresh;
      ++n_cow;
      bm->drop(old);
      s.table.back() = fresh;
    }
    slots_out[i] = static_cast<int64_t>(s.table.back()) * bm->block_size + row;
    ++s.len;
  }
  *n_cow_out = n_cow;
  for (int i = 0; i < n; ++i) {
    pkv_bm::Seq& s = *seqs[i];
    if (!tokens) {
      s.tracked = false;
      s.partial.clear();
      continue;
    }
    if (!s.tracked) continue;
    s.partial.push_back(tokens[i]);
    if (static_cast<int>(s.partial.size()) < bm->block_size) continue;
    // the token completed its block: register it under the chain hash, as a prompt block is
    s.parent = block_hash(s.parent, s.partial.data(), bm->block_size);
    s.partial.clear();
    const int32_t b = s.table.back();
    if (!bm->registered[b] && !bm->cached.count(s.parent)) {
      bm->cached.emplace(s.parent, b);
      bm->block_hash_of[b] = s.parent;
      bm->registered[b] = 1;
    }
  }
  return PKV_OK;
}

extern "C" int pkv_bm_append_slots(pkv_bm* bm, const int64_t* seq_ids, int n, int64_t* slots_out,
                                   int64_t* cow_pairs_out, int* n_cow_out) {
  return append_impl(bm, seq_ids, nullptr, n, slots_out, cow_pairs_out, n_cow_out);
}

extern "C" int pkv_bm_append_tokens(pkv_bm* bm, const int64_t* seq_ids, const int32_t* tokens, int n,
                                    int64_t* slots_out, int64_t* cow_pairs_out, int* n_cow_out) {
  if (n > 0 && !tokens) return set_error(PKV_ERR_INVALID, "pkv_bm_append_tokens: null tokens");
  return append_impl(bm, seq_ids, n > 0 ? tokens : nullptr, n, slots_out, cow_pairs_out, n_cow_out);
}

extern "C" int pkv_bm_slots(const pkv_bm* bm, int64_t seq_id, int start, int count, int64_t* slots_out) {
  if (!bm || start < 0 || count < 0 || (count > 0 && !slots_out))
    return set_error(PKV_ERR_INVALID, "pkv_bm_slots: bad arguments");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end() || it->second.swapped || static_cast<int64_t>(start) + count > it->second.len)
    return set_error(PKV_ERR_INVALID, "pkv_bm_slots: unknown or swapped-out sequence, or range past its length");
  const auto& table = it->second.table;
  for (int i = 0; i < count; ++i) {
    int p = start + i;
    slots_out[i] = static_cast<int64_t>(table[p / bm->block_size]) * bm->block_size + p % bm->block_size;
  }
  return PKV_OK;
}

extern "C" int pkv_bm_free_seq(pkv_bm* bm, int64_t seq_id) {
  if (!bm) return set_error(PKV_ERR_INVALID, "pkv_bm_free_seq: null manager");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return set_error(PKV_ERR_INVALID, "pkv_bm_free_seq: unknown sequence %lld", (long long)seq_id);
  if (it->second.swapped) {
    for (int32_t b : it->second.table) bm->host_drop(b);
  } else {
    for (int32_t b : it->second.table) bm->drop(b);
  }
  bm->seqs.erase(it);
  return PKV_OK;
}

extern "C" int pkv_bm_seq_len(const pkv_bm* bm, int64_t seq_id) {
  if (!bm) return set_error(PKV_ERR_INVALID, "pkv_bm_seq_len: null manager");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return set_error(PKV_ERR_INVALID, "pkv_bm_seq_len: unknown sequence");
  return it->second.len;
}

extern "C" int pkv_bm_seq_blocks(const pkv_bm* bm, int64_t seq_id) {
  if (!bm) return set_error(PKV_ERR_INVALID, "pkv_bm_seq_blocks: null manager");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return set_error(PKV_ERR_INVALID, "pkv_bm_seq_blocks: unknown sequence");
  return static_cast<int>(it->second.table.size());
}

extern "C" int pkv_bm_export_tables(const pkv_bm* bm, const int64_t* seq_ids, int n, int32_t* tables,
                                    int max_blocks, int32_t* context_lens) {
  if (!bm || n < 0 || max_blocks < 0 || (n > 0 && (!seq_ids || !context_lens || (max_blocks > 0 && !tables))))
    return set_error(PKV_ERR_INVALID, "pkv_bm_export_tables: bad arguments");
  std::vector<const pkv_bm::Seq*> seqs(static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end() || it->second.swapped || static_cast<int>(it->second.table.size()) > max_blocks)
      return set_error(PKV_ERR_INVALID, "pkv_bm_export_tables: unknown sequence %lld or table longer than %d",
                       (long long)seq_ids[i], max_blocks);
    seqs[i] = &it->second;
  }
  for (int i = 0; i < n; ++i) {
    const auto& s = *seqs[i];
    int32_t* row = tables + static_cast<size_t>(i) * max_blocks;
    std::copy(s.table.begin(), s.table.end(), row);
    std::fill(row + s.table.size(), row + max_blocks, 0);
    context_lens[i] = s.len;
  }
  return PKV_OK;
}

// ---- swap space ------------------------------------------------------------------

extern "C" pkv_bm* pkv_bm_create_with_swap_space(int num_blocks, int block_size, const int32_t* initial_order,
                                                 int num_host_blocks) {
  if (num_host_blocks < 0) {
    set_error(PKV_ERR_INVALID, "pkv_bm_create_with_swap_space: negative host pool");
    return nullptr;
  }
  pkv_bm* bm = pkv_bm_create(num_blocks, block_size, initial_order);
  if (!bm) return nullptr;
  bm->num_host_blocks = num_host_blocks;
  bm->host_ref.assign(num_host_blocks, 0);
  for (int i = 0; i < num_host_blocks; ++i) bm->host_free.push_back(i);
  return bm;
}

extern "C" int pkv_bm_num_host_free(const pkv_bm* bm) {
  return bm ? static_cast<int>(bm->host_free.size()) : PKV_ERR_INVALID;
}

extern "C" int pkv_bm_host_refcount(const pkv_bm* bm, int32_t block) {
  if (!bm || block < 0 || block >= bm->num_host_blocks)
    return set_error(PKV_ERR_INVALID, "pkv_bm_host_refcount: bad host block %d", block);
  return bm->host_ref[block];
}

extern "C" int pkv_bm_is_swapped(const pkv_bm* bm, int64_t seq_id) {
  if (!bm) return set_error(PKV_ERR_INVALID, "pkv_bm_is_swapped: null manager");
  auto it = bm->seqs.find(seq_id);
  if (it == bm->seqs.end()) return set_error(PKV_ERR_INVALID, "pkv_bm_is_swapped: unknown sequence");
  return it->second.swapped ? 1 : 0;
}

// Shared by swap_out (device -> host) and swap_in (host -> device).
static int swap_move(pkv_bm* bm, const int64_t* seq_ids, int n, int64_t* pairs_out, int cap, int* n_pairs_out,
                     bool out, const char* what) {
  if (!bm || n < 0 || (n > 0 && !seq_ids) || !n_pairs_out || cap < 0 || (cap > 0 && !pairs_out))
    return set_error(PKV_ERR_INVALID, "%s: bad arguments", what);
  *n_pairs_out = 0;
  std::vector<pkv_bm::Seq*> seqs(n);
  std::unordered_map<int64_t, int> seen;
  for (int i = 0; i < n; ++i) {
    auto it = bm->seqs.find(seq_ids[i]);
    if (it == bm->seqs.end() || it->second.swapped == out || !seen.emplace(seq_ids[i], i).second)
      return set_error(PKV_ERR_INVALID, "%s: sequence %lld unknown, repeated or in the wrong pool", what,
                       (long long)seq_ids[i]);
    seqs[i] = &it->second;
  }
  std::unordered_map<int32_t, int32_t> mapping;  // source block -> destination block
  int distinct = 0;
  {
    std::unordered_map<int32_t, char> marked;
    for (auto* s : seqs)
      for (int32_t b : s->table)
        if (marked.emplace(b, 1).second) ++distinct;
  }
  const int avail = out ? static_cast<int>(bm->host_free.size()) : bm->free_list.size();
  if (distinct > avail)
    return set_error(PKV_ERR_OOM, "%s: %s pool exhausted (%d blocks needed, %d free)", what, out ? "host" : "device",
                     distinct, avail);
  if (distinct > cap) return set_error(PKV_ERR_INVALID, "%s: pair buffer holds %d pairs, %d needed", what, cap, distinct);
  int np = 0;
  for (auto* s : seqs) {
    for (int32_t& b : s->table) {
      auto m = mapping.find(b);
      int32_t d;
      if (m != mapping.end()) {
        d = m->second;
        if (out) ++bm->host_ref[d]; else ++bm->ref[d];
      } else {
        if (out) {
          d = bm->host_free.front();
          bm->host_free.pop_front();
          bm->host_ref[d] = 1;
        } else {
          d = bm->take();
        }
        mapping.emplace(b, d);
        pairs_out[2 * np] = b;
        pairs_out[2 * np + 1] = d;
        ++np;
      }
      if (out) bm->drop(b); else bm->host_drop(b);
      b = d;
    }
    s->swapped = out;
  }
  *n_pairs_out = np;
  return PKV_OK;
}

extern "C" int pkv_bm_swap_out(pkv_bm* bm, const int64_t* seq_ids, int n, int64_t* pairs_out, int cap,
                               int* n_pairs_out) {
  return swap_move(bm, seq_ids, n, pairs_out, cap, n_pairs_out, true, "pkv_bm_swap_out");
}

extern "C" int pkv_bm_swap_in(pkv_bm* bm, const int64_t* seq_ids, int n, int64_t* pairs_out, int cap,
                              int* n_pairs_out) {
  return swap_move(bm, seq_ids, n, pairs_out, cap, n_pairs_out, false, "pkv_bm_swap_in");
}

// ---- automatic prefix caching ------------------------------------------------------

extern "C" int pkv_bm_num_cached_blocks(const pkv_bm* bm) {
  return bm ? static_cast<int>(bm->cached.size()) : PKV_ERR_INVALID;
}

extern "C" int pkv_bm_add_seq_tokens(pkv_bm* bm, int64_t seq_id, const int32_t* tokens, int num_tokens,
                                     int* cached_tokens_out) {
  if (!bm || num_tokens < 0 || (num_tokens > 0 && !tokens) || !cached_tokens_out)
    return set_error(PKV_ERR_INVALID, "pkv_bm_add_seq_tokens: bad arguments");
  if (bm->seqs.count(seq_id))
    return set_error(PKV_ERR_INVALID, "pkv_bm_add_seq_tokens: sequence %lld exists", (long long)seq_id);
  const int bs = bm->block_size;
  const int nfull = num_tokens / bs;
  std::vector<uint64_t> hashes(nfull);
  uint64_t parent = 0;
  for (int i = 0; i < nfull; ++i) hashes[i] = parent = block_hash(parent, tokens + static_cast<size_t>(i) * bs, bs);
  // the block holding the last token is never taken from the cache
  const int cap = num_tokens > 0 ? (num_tokens - 1) / bs : 0;
  std::vector<int32_t> hits;
  for (int i = 0; i < cap; ++i) {
    auto it = bm->cached.find(hashes[i]);
    if (it == bm->cached.end()) break;
    hits.push_back(it->second);
  }
  int revive = 0;
  for (int32_t b : hits) revive += bm->ref[b] == 0;
  const int total = bm->blocks_for(num_tokens);
  const int fresh = total - static_cast<int>(hits.size());
  if (fresh > bm->free_list.size() - revive)
    return set_error(PKV_ERR_OOM, "pkv_bm_add_seq_tokens: pool exhausted (%d fresh blocks needed)", fresh);
  pkv_bm::Seq seq;
  seq.table.reserve(total);
  for (int32_t b : hits) {
    if (bm->ref[b] == 0) {
      bm->free_list.remove(b);
      bm->ref[b] = 1;
    } else {
      ++bm->ref[b];
    }
    seq.table.push_back(b);
  }
  for (int i = static_cast<int>(hits.size()); i < total; ++i) {
    const int32_t b = bm->take();
    seq.table.push_back(b);
    if (i < nfull && !bm->cached.count(hashes[i])) {
      bm->cached.emplace(hashes[i], b);
      bm->block_hash_of[b] = hashes[i];
      bm->registered[b] = 1;
    }
  }
  seq.len = num_tokens;
  seq.tracked = true;
  seq.parent = nfull > 0 ? hashes[nfull - 1] : 0;
  seq.partial.assign(tokens + static_cast<size_t>(nfull) * bs, tokens + num_tokens);
  bm->seqs.emplace(seq_id, std::move(seq));
  *cached_tokens_out = static_cast<int>(hits.size()) * bs;
  return PKV_OK;
}
