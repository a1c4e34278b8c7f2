"""Oracle: reference model of the block allocator and per-sequence block tables.

TEST INFRASTRUCTURE ONLY -- see the package docstring.

What it follows
  * Outcome School explainer, "vLLM的核心创新：PagedAttention": fixed-size blocks, a
    new block only when a request needs more room, blocks need not be contiguous,
    a per-request block table keeps their order, and every block of a finished
    request goes straight back to the shared pool, where any request can take it.
  * Same page, "内存共享": requests with an identical prefix point their tables at the
    same physical blocks; beams share blocks up to the point where they diverge.
  * vLLM 初探 §1.4: the block-table figure (logical Block i -> physical block).

Rules the pages leave open (readings):
  * The free list is a FIFO queue.  Its initial order is an input (a seeded
    permutation drawn by the workload generator); freed blocks join the back in
    the order they appear in the freed table.
  * Every block has a reference count = number of tables holding it.
  * append_slots, per sequence in call order: if the next position starts a new
    block (position % bs == 0) take a fresh block; else, if the last block is
    shared (refcount > 1), take a fresh block, record (old, new) as a copy-on-write
    pair, drop one reference to old and put new in its place.  The call is
    all-or-nothing: if the pool cannot cover every allocation, nothing changes.
  * fork(parent, child) gives the child a copy of the parent's table and length and
    one more reference on every block.
  * add_seq with shared prefix blocks: they must be full blocks; the remaining
    blocks are taken fresh (all-or-nothing).

Swap space (intelliparadigm article, §4.2 OOM错误: swap_space extends the pool into
host memory).  Readings:
  * A second pool of host blocks with its own FIFO free list (initial order 0..H-1)
    and reference counts.
  * swap_out(seqs) moves the listed sequences' tables to host blocks: every distinct
    device block among them (in order of first appearance, sequence by sequence)
    gets one host block, the pair (device, host) is returned for the copy, the
    table entry becomes the host block and the device block loses one reference.
    swap_in(seqs) is the mirror image.  Both are all-or-nothing.  A swapped-out
    sequence can only be swapped in or freed.

Automatic prefix caching (Outcome School explainer, "内存共享": requests with an
identical prefix, e.g. one long system prompt, keep a single copy of its blocks;
vLLM 初探 §1.4: shared system prompts save 30-50% of the memory).  Readings:
  * A full block is identified by the chain hash h_i = FNV-1a-64 of the 8
    little-endian bytes of h_(i-1) (h_(-1) = 0) followed by the block's token ids
    as 4-byte little-endian integers.  FNV-1a-64: start from 0xcbf29ce484222325;
    per byte, xor it in, then multiply by 0x100000001b3 modulo 2^64.
  * add_seq_tokens(seq, tokens) takes the longest run of leading blocks whose hashes
    are registered, but never the block holding the last token (that token is
    always computed again), so at most (n - 1) // bs blocks.  Blocks taken from
    the cache gain a reference; a cached block with no references is taken back
    out of the free list.  The other blocks are fresh; each fresh FULL block
    registers its hash unless the hash is already registered.
  * A registered block whose references drop to zero stays registered while it
    waits in the free list; when the free list hands it out again its
    registration is dropped (eviction in free-list order).
  * Blocks filled during decode: a sequence created by add_seq_tokens keeps its
    token history (the chain hash of its last full block and the ids of the block
    being filled); fork copies it.  append_tokens(seqs, tokens) is append_slots
    plus one token id per sequence: when a token completes its sequence's block,
    the block registers under its chain hash like a full prompt block (unless the
    hash is already registered; sequences in call order).  append_slots, which
    carries no ids, ends a sequence's history; add_seq sequences have none.

Parity status: pinned (invariants, the pages' block-table example, hand-worked
copy-on-write, swap and prefix-cache cases, FNV-1a test vectors).
"""
from __future__ import annotations

from collections import deque

OK = 0
ERR_INVALID = -1
ERR_OOM = -2


class BlockManagerError(Exception):
    def __init__(self, code: int, msg: str):
        super().__init__(msg)
        self.code = code


FNV_OFFSET = 0xCBF29CE484222325
FNV_PRIME = 0x100000001B3


def fnv1a64(data: bytes, h: int = FNV_OFFSET) -> int:
    for byte in data:
        h ^= byte
        h = (h * FNV_PRIME) & 0xFFFFFFFFFFFFFFFF
    return h


def block_hash(parent: int, tokens) -> int:
    data = int(parent).to_bytes(8, "little") + b"".join(int(t).to_bytes(4, "little", signed=True) for t in tokens)
    return fnv1a64(data)


class BlockManagerModel:
    def __init__(self, num_blocks: int, block_size: int, initial_order=None, num_host_blocks: int = 0):
        if num_blocks <= 0 or block_size <= 0 or num_host_blocks < 0:
            raise BlockManagerError(ERR_INVALID, "bad sizes")
        order = list(range(num_blocks)) if initial_order is None else [int(b) for b in initial_order]
        if sorted(order) != list(range(num_blocks)):
            raise BlockManagerError(ERR_INVALID, "initial order is not a permutation")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = deque(order)
        self.ref = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        self.host_free = deque(range(num_host_blocks))
        self.host_ref = [0] * num_host_blocks
        self.swapped: set[int] = set()
        self.cached: dict[int, int] = {}        # hash -> device block
        self.block_hash: dict[int, int] = {}    # device block -> its registered hash
        self.hist: dict[int, tuple | None] = {}  # seq -> (parent hash, partial token ids) or None

    # -- blocks -------------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free)

    def alloc(self) -> int:
        if not self.free:
            raise BlockManagerError(ERR_OOM, "pool exhausted")
        b = self.free.popleft()
        self.ref[b] = 1
        h = self.block_hash.pop(b, None)        # handing a cached block out evicts it
        if h is not None:
            del self.cached[h]
        return b

    def _check_block(self, b: int):
        if not (0 <= b < self.num_blocks):
            raise BlockManagerError(ERR_INVALID, f"block {b} out of range")

    def incref(self, b: int):
        self._check_block(b)
        if self.ref[b] <= 0:
            raise BlockManagerError(ERR_INVALID, f"block {b} is free")
        self.ref[b] += 1

    def decref(self, b: int):
        self._check_block(b)
        if self.ref[b] <= 0:
            raise BlockManagerError(ERR_INVALID, f"block {b} is already free")
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free.append(b)

    def refcount(self, b: int) -> int:
        self._check_block(b)
        return self.ref[b]

    # -- sequences ----------------------------------------------------------
    def _blocks_for(self, num_tokens: int) -> int:
        return -(-num_tokens // self.block_size)

    def add_seq(self, seq_id: int, num_tokens: int, shared_prefix_blocks=()):
        shared = [int(b) for b in shared_prefix_blocks]
        if seq_id in self.tables or num_tokens < 0:
            raise BlockManagerError(ERR_INVALID, "bad sequence")
        if len(shared) * self.block_size > num_tokens:
            raise BlockManagerError(ERR_INVALID, "shared prefix longer than the sequence")
        for b in shared:
            self._check_block(b)
            if self.ref[b] <= 0:
                raise BlockManagerError(ERR_INVALID, "shared block is free")
        fresh = self._blocks_for(num_tokens) - len(shared)
        if fresh > len(self.free):
            raise BlockManagerError(ERR_OOM, "pool exhausted")
        for b in shared:
            self.ref[b] += 1
        table = shared + [self.alloc() for _ in range(fresh)]
        self.tables[seq_id] = table
        self.lens[seq_id] = num_tokens
        self.hist[seq_id] = None

    def fork(self, parent: int, child: int):
        if parent not in self.tables or child in self.tables or parent in self.swapped:
            raise BlockManagerError(ERR_INVALID, "bad fork")
        table = list(self.tables[parent])
        for b in table:
            self.ref[b] += 1
        self.tables[child] = table
        self.lens[child] = self.lens[parent]
        h = self.hist.get(parent)
        self.hist[child] = None if h is None else (h[0], list(h[1]))

    def append_slots(self, seq_ids):
        """One new token per listed sequence; returns (slots, cow_pairs).  The
        sequences' token histories end (nothing they fill later registers)."""
        slots, pairs = self._append(seq_ids)
        for s in seq_ids:
            self.hist[int(s)] = None
        return slots, pairs

    def append_tokens(self, seq_ids, tokens):
        """append_slots with the token id of each new position; a tracked sequence
        registers the block a token completes under its chain hash."""
        seq_ids = [int(s) for s in seq_ids]
        tokens = [int(t) for t in tokens]
        if len(tokens) != len(seq_ids):
            raise BlockManagerError(ERR_INVALID, "one token per sequence")
        slots, pairs = self._append(seq_ids)
        for s, tok in zip(seq_ids, tokens):
            h = self.hist.get(s)
            if h is None:
                continue
            parent, partial = h
            partial = partial + [tok]
            if len(partial) == self.block_size:
                parent = block_hash(parent, partial)
                partial = []
                b = self.tables[s][-1]
                if b not in self.block_hash and parent not in self.cached:
                    self.cached[parent] = b
                    self.block_hash[b] = parent
            self.hist[s] = (parent, partial)
        return slots, pairs

    def _append(self, seq_ids):
        seq_ids = [int(s) for s in seq_ids]
        if (len(set(seq_ids)) != len(seq_ids) or any(s not in self.tables for s in seq_ids)
                or any(s in self.swapped for s in seq_ids)):
            raise BlockManagerError(ERR_INVALID, "unknown, repeated or swapped-out sequence")
        # Dry run: count fresh blocks, following the reference counts as they change.
        need = 0
        pending = {}
        for s in seq_ids:
            pos = self.lens[s]
            if pos % self.block_size == 0:
                need += 1
            else:
                last = self.tables[s][-1]
                if self.ref[last] + pending.get(last, 0) > 1:
                    need += 1
                    pending[last] = pending.get(last, 0) - 1
        if need > len(self.free):
            raise BlockManagerError(ERR_OOM, "pool exhausted")
        slots, pairs = [], []
        for s in seq_ids:
            pos = self.lens[s]
            table = self.tables[s]
            if pos % self.block_size == 0:
                table.append(self.alloc())
            elif self.ref[table[-1]] > 1:
                old = table[-1]
                new = self.alloc()
                pairs.append((old, new))
                self.decref(old)
                table[-1] = new
            slots.append(table[-1] * self.block_size + pos % self.block_size)
            self.lens[s] = pos + 1
        return slots, pairs

    def slots(self, seq_id: int, start: int, count: int):
        """Slots of positions start .. start+count-1 of an existing sequence."""
        if (seq_id not in self.tables or seq_id in self.swapped or start < 0 or count < 0
                or start + count > self.lens[seq_id]):
            raise BlockManagerError(ERR_INVALID, "bad range")
        table = self.tables[seq_id]
        return [table[p // self.block_size] * self.block_size + p % self.block_size
                for p in range(start, start + count)]

    def free_seq(self, seq_id: int):
        if seq_id not in self.tables:
            raise BlockManagerError(ERR_INVALID, "unknown sequence")
        table = self.tables.pop(seq_id)
        if seq_id in self.swapped:
            self.swapped.discard(seq_id)
            for b in table:
                self._host_decref(b)
        else:
            for b in table:
                self.decref(b)
        del self.lens[seq_id]
        self.hist.pop(seq_id, None)

    def export_tables(self, seq_ids, max_blocks: int):
        tables = []
        lens = []
        for s in seq_ids:
            if s not in self.tables or s in self.swapped or len(self.tables[s]) > max_blocks:
                raise BlockManagerError(ERR_INVALID, "unknown sequence or table too long")
            row = list(self.tables[s]) + [0] * (max_blocks - len(self.tables[s]))
            tables.append(row)
            lens.append(self.lens[s])
        return tables, lens

    def seq_len(self, seq_id: int) -> int:
        return self.lens[seq_id]

    # -- swap space -----------------------------------------------------------
    def num_host_free(self) -> int:
        return len(self.host_free)

    def host_refcount(self, b: int) -> int:
        return self.host_ref[b]

    def is_swapped(self, seq_id: int) -> bool:
        return seq_id in self.swapped

    def _host_decref(self, b: int):
        self.host_ref[b] -= 1
        if self.host_ref[b] == 0:
            self.host_free.append(b)

    def _check_swap_ids(self, seq_ids, want_swapped: bool):
        if len(set(seq_ids)) != len(seq_ids):
            raise BlockManagerError(ERR_INVALID, "repeated sequence")
        for s in seq_ids:
            if s not in self.tables or (s in self.swapped) != want_swapped:
                raise BlockManagerError(ERR_INVALID, "sequence in the wrong place")

    def _distinct_blocks(self, seq_ids):
        seen = []
        marked = set()
        for s in seq_ids:
            for b in self.tables[s]:
                if b not in marked:
                    marked.add(b)
                    seen.append(b)
        return seen

    def swap_out(self, seq_ids):
        """Move the listed resident sequences to host blocks; returns (device, host) pairs."""
        seq_ids = [int(s) for s in seq_ids]
        self._check_swap_ids(seq_ids, want_swapped=False)
        if len(self._distinct_blocks(seq_ids)) > len(self.host_free):
            raise BlockManagerError(ERR_OOM, "host pool exhausted")
        mapping, pairs = {}, []
        for s in seq_ids:
            table = self.tables[s]
            for j, b in enumerate(table):
                if b in mapping:
                    self.host_ref[mapping[b]] += 1
                else:
                    hb = self.host_free.popleft()
                    self.host_ref[hb] = 1
                    mapping[b] = hb
                    pairs.append((b, hb))
                table[j] = mapping[b]
                self.decref(b)
            self.swapped.add(s)
        return pairs

    def swap_in(self, seq_ids):
        """Bring the listed swapped-out sequences back; returns (host, device) pairs."""
        seq_ids = [int(s) for s in seq_ids]
        self._check_swap_ids(seq_ids, want_swapped=True)
        if len(self._distinct_blocks(seq_ids)) > len(self.free):
            raise BlockManagerError(ERR_OOM, "pool exhausted")
        mapping, pairs = {}, []
        for s in seq_ids:
            table = self.tables[s]
            for j, hb in enumerate(table):
                if hb in mapping:
                    self.ref[mapping[hb]] += 1
                else:
                    mapping[hb] = self.alloc()
                    pairs.append((hb, mapping[hb]))
                table[j] = mapping[hb]
                self._host_decref(hb)
            self.swapped.discard(s)
        return pairs

    # -- automatic prefix caching ---------------------------------------------
    def num_cached_blocks(self) -> int:
        return len(self.cached)

    def add_seq_tokens(self, seq_id: int, tokens) -> int:
        """New sequence from its prompt token ids; returns the number of leading
        tokens whose K/V came from cached blocks."""
        tokens = [int(t) for t in tokens]
        n = len(tokens)
        bs = self.block_size
        if seq_id in self.tables:
            raise BlockManagerError(ERR_INVALID, "bad sequence")
        hashes = []
        parent = 0
        for i in range(n // bs):
            parent = block_hash(parent, tokens[i * bs:(i + 1) * bs])
            hashes.append(parent)
        cap = (n - 1) // bs if n > 0 else 0
        hits = []
        for i in range(cap):
            b = self.cached.get(hashes[i])
            if b is None:
                break
            hits.append(b)
        revive = sum(1 for b in hits if self.ref[b] == 0)
        fresh = self._blocks_for(n) - len(hits)
        if fresh > len(self.free) - revive:
            raise BlockManagerError(ERR_OOM, "pool exhausted")
        for b in hits:
            if self.ref[b] == 0:
                self.free.remove(b)
                self.ref[b] = 1
            else:
                self.ref[b] += 1
        table = list(hits)
        for i in range(len(hits), self._blocks_for(n)):
            b = self.alloc()
            table.append(b)
            if i < len(hashes) and hashes[i] not in self.cached:
                self.cached[hashes[i]] = b
                self.block_hash[b] = hashes[i]
        self.tables[seq_id] = table
        self.lens[seq_id] = n
        self.hist[seq_id] = (hashes[-1] if hashes else 0, tokens[len(hashes) * bs:])
        return len(hits) * bs
