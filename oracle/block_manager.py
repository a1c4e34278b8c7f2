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

Parity status: pinned (invariants, the pages' block-table example, hand-worked
copy-on-write cases).
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


class BlockManagerModel:
    def __init__(self, num_blocks: int, block_size: int, initial_order=None):
        if num_blocks <= 0 or block_size <= 0:
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

    # -- blocks -------------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free)

    def alloc(self) -> int:
        if not self.free:
            raise BlockManagerError(ERR_OOM, "pool exhausted")
        b = self.free.popleft()
        self.ref[b] = 1
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

    def fork(self, parent: int, child: int):
        if parent not in self.tables or child in self.tables:
            raise BlockManagerError(ERR_INVALID, "bad fork")
        table = list(self.tables[parent])
        for b in table:
            self.ref[b] += 1
        self.tables[child] = table
        self.lens[child] = self.lens[parent]

    def append_slots(self, seq_ids):
        """One new token per listed sequence; returns (slots, cow_pairs)."""
        seq_ids = [int(s) for s in seq_ids]
        if len(set(seq_ids)) != len(seq_ids) or any(s not in self.tables for s in seq_ids):
            raise BlockManagerError(ERR_INVALID, "unknown or repeated sequence")
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
        if seq_id not in self.tables or start < 0 or count < 0 or start + count > self.lens[seq_id]:
            raise BlockManagerError(ERR_INVALID, "bad range")
        table = self.tables[seq_id]
        return [table[p // self.block_size] * self.block_size + p % self.block_size
                for p in range(start, start + count)]

    def free_seq(self, seq_id: int):
        if seq_id not in self.tables:
            raise BlockManagerError(ERR_INVALID, "unknown sequence")
        for b in self.tables.pop(seq_id):
            self.decref(b)
        del self.lens[seq_id]

    def export_tables(self, seq_ids, max_blocks: int):
        tables = []
        lens = []
        for s in seq_ids:
            if s not in self.tables or len(self.tables[s]) > max_blocks:
                raise BlockManagerError(ERR_INVALID, "unknown sequence or table too long")
            row = list(self.tables[s]) + [0] * (max_blocks - len(self.tables[s]))
            tables.append(row)
            lens.append(self.lens[s])
        return tables, lens

    def seq_len(self, seq_id: int) -> int:
        return self.lens[seq_id]
