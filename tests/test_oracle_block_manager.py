"""Pins for the block-allocator reference model (CPU only).

The model is pinned to the pages' block-table figure (vLLM 初探 §1.4), to
hand-worked copy-on-write cases, and to invariants that hold after any sequence
of operations: every table entry is one reference, free + live blocks = pool,
a free block never sits in a live table, and a table always has
ceil(length / block_size) entries.
"""
import json
import os

import numpy as np
import pytest

import workloads as wl
from oracle.block_manager import (ERR_INVALID, ERR_OOM, BlockManagerError, BlockManagerModel, block_hash,
                                  fnv1a64)


def check_invariants(m: BlockManagerModel):
    refs = [0] * m.num_blocks
    host_refs = [0] * len(m.host_ref)
    for s, table in m.tables.items():
        for b in table:
            if s in m.swapped:
                host_refs[b] += 1
            else:
                refs[b] += 1
    assert refs == m.ref, "reference counts must equal the number of table entries"
    assert host_refs == m.host_ref, "host reference counts must equal the swapped-out table entries"
    live = {b for b in range(m.num_blocks) if m.ref[b] > 0}
    assert len(m.free) + len(live) == m.num_blocks
    assert not (set(m.free) & live)
    assert len(set(m.free)) == len(m.free)
    host_live = {b for b in range(len(m.host_ref)) if m.host_ref[b] > 0}
    assert len(m.host_free) + len(host_live) == len(m.host_ref)
    assert not (set(m.host_free) & host_live)
    for s, table in m.tables.items():
        assert len(table) == -(-m.lens[s] // m.block_size)
    # the prefix cache maps each registered hash to one block and back
    assert len(m.cached) == len(m.block_hash)
    for h, b in m.cached.items():
        assert m.block_hash[b] == h


def test_block_table_figure():
    fig = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "block_table_figure.json")))
    sc, ex = fig["scenario"], fig["expected"]
    m = BlockManagerModel(8, sc["block_size"], sc["initial_free_order"])
    A, B = 1, 2
    m.add_seq(A, 16)
    m.add_seq(B, 16)
    for _ in range(16):
        m.append_slots([A])
    for _ in range(16):
        m.append_slots([B])
    assert m.tables[A] == ex["table_A"] == [fig["printed"]["logical_table"]["Block 0"],
                                            fig["printed"]["logical_table"]["Block 1"]]
    assert m.tables[B] == ex["table_B"]
    assert sorted(m.free) == ex["free_after"] == fig["printed"]["free_blocks"]
    for pos, slot in ex["slots_A_positions"].items():
        assert m.slots(A, int(pos), 1) == [slot]
    for pos, slot in ex["slots_B_positions"].items():
        assert m.slots(B, int(pos), 1) == [slot]
    check_invariants(m)


def test_blocks_return_to_pool_on_finish():
    """Outcome School explainer: a finished request's blocks go straight back to the pool."""
    m = BlockManagerModel(10, 4, list(range(10)))
    m.add_seq(0, 9)          # blocks 0,1,2
    m.add_seq(1, 4)          # block 3
    assert m.num_free() == 6
    m.free_seq(0)
    assert list(m.free) == [4, 5, 6, 7, 8, 9, 0, 1, 2]
    m.add_seq(2, 20)         # takes 5 blocks from the front
    assert m.tables[2] == [4, 5, 6, 7, 8]
    check_invariants(m)


def test_new_block_only_when_last_is_full():
    m = BlockManagerModel(6, 4)
    m.add_seq(7, 0)
    slots_seen = []
    for _ in range(9):
        slots, pairs = m.append_slots([7])
        slots_seen += slots
        assert pairs == []
    assert m.tables[7] == [0, 1, 2]
    assert slots_seen == [0, 1, 2, 3, 4, 5, 6, 7, 8]
    assert m.num_free() == 3


def test_beam_fork_copy_on_write_by_hand():
    """Four beams share a partial last block; appending in id order, beams 0-2 copy
    it and beam 3, by then its only holder, writes in place."""
    m = BlockManagerModel(16, 4, list(range(16)))
    m.add_seq(0, 6)                      # blocks [0, 1], last block has 2 of 4 rows
    for child in (1, 2, 3):
        m.fork(0, child)
    assert m.ref[0] == 4 and m.ref[1] == 4
    slots, pairs = m.append_slots([0, 1, 2, 3])
    assert pairs == [(1, 2), (1, 3), (1, 4)]
    assert [m.tables[s] for s in range(4)] == [[0, 2], [0, 3], [0, 4], [0, 1]]
    assert slots == [2 * 4 + 2, 3 * 4 + 2, 4 * 4 + 2, 1 * 4 + 2]
    assert m.ref[0] == 4 and m.ref[1] == 1
    check_invariants(m)


def test_fork_at_block_boundary_needs_no_copy():
    m = BlockManagerModel(8, 4, list(range(8)))
    m.add_seq(0, 8)                      # two full blocks
    m.fork(0, 1)
    slots, pairs = m.append_slots([0, 1])
    assert pairs == [] and slots == [2 * 4, 3 * 4]
    assert m.tables[0][:2] == m.tables[1][:2] == [0, 1]
    check_invariants(m)


def test_shared_prefix_refcounts():
    """Outcome School explainer, "内存共享": identical prefixes stored once."""
    m = BlockManagerModel(400, 16, list(range(400)))
    m.add_seq(0, 1024 + 30)
    prefix = m.tables[0][:64]
    for s in range(1, 128):
        m.add_seq(s, 1024 + s % 16 + 1, prefix)
    assert all(m.ref[b] == 128 for b in prefix)
    assert all(m.tables[s][:64] == prefix for s in range(128))
    check_invariants(m)
    for s in range(128):
        m.free_seq(s)
    assert m.num_free() == 400 and sum(m.ref) == 0


def test_oom_is_all_or_nothing():
    m = BlockManagerModel(3, 4, [2, 0, 1])
    m.add_seq(0, 4)
    m.add_seq(1, 4)
    before = (list(m.free), dict((k, list(v)) for k, v in m.tables.items()), dict(m.lens), list(m.ref))
    with pytest.raises(BlockManagerError) as e:
        m.append_slots([0, 1])           # both need a new block, only one is free
    assert e.value.code == ERR_OOM
    assert before == (list(m.free), dict((k, list(v)) for k, v in m.tables.items()), dict(m.lens), list(m.ref))
    with pytest.raises(BlockManagerError) as e:
        m.add_seq(2, 9)
    assert e.value.code == ERR_OOM


def test_invalid_operations():
    m = BlockManagerModel(4, 4)
    m.add_seq(0, 3)
    for call in (lambda: m.add_seq(0, 1), lambda: m.fork(5, 6), lambda: m.fork(0, 0),
                 lambda: m.append_slots([0, 0]), lambda: m.append_slots([9]),
                 lambda: m.free_seq(3), lambda: m.decref(3), lambda: m.incref(2),
                 lambda: m.slots(0, 2, 2), lambda: m.add_seq(1, 3, [0, 1])):
        with pytest.raises(BlockManagerError) as e:
            call()
        assert e.value.code == ERR_INVALID


def check_histories(m: BlockManagerModel, texts):
    """A sequence with a known token text holds the chain hash of its full blocks and the
    ids of its partial block; one without holds none."""
    bs = m.block_size
    for s in m.tables:
        txt = texts.get(s)
        if txt is None:
            assert m.hist[s] is None
            continue
        assert len(txt) == m.lens[s]
        nf = len(txt) // bs
        parent = 0
        for i in range(nf):
            parent = block_hash(parent, txt[i * bs:(i + 1) * bs])
        assert m.hist[s] == (parent, txt[nf * bs:])


def random_ops(seed, steps=400, num_blocks=48, block_size=4, extended=False):
    """A seeded random mix of every operation; checks invariants after each one.
    ``extended`` adds swap-out / swap-in, prompt-token (prefix-cached) admission,
    decode appends with token ids, and prompts that continue a generated text."""
    rng = wl.rng_for(seed)
    m = BlockManagerModel(num_blocks, block_size, rng.permutation(num_blocks),
                          num_host_blocks=num_blocks // 2 if extended else 0)
    prompts = [list(rng.integers(0, 5, size=40)) for _ in range(3)]   # few distinct prompts: many hits
    texts = {}  # seq -> its token ids, or None when unknown
    next_id = 0
    for _ in range(steps):
        op = rng.integers(0, 10 if extended else 5)
        live = sorted(s for s in m.tables if s not in m.swapped)
        gone = sorted(m.swapped)
        try:
            if op == 8:
                if live:
                    pick = [int(x) for x in rng.permutation(live)[:rng.integers(1, len(live) + 1)]]
                    toks = [int(t) for t in rng.integers(0, 5, size=len(pick))]
                    m.append_tokens(pick, toks)
                    for s_, t_ in zip(pick, toks):
                        if texts.get(s_) is not None:
                            texts[s_] = texts[s_] + [t_]
                continue
            if op == 9:
                known = [x for x in live if texts.get(x) is not None]
                if known:
                    src = known[rng.integers(len(known))]
                    prompt = texts[src] + [int(t) for t in rng.integers(0, 5, size=int(rng.integers(1, 4)))]
                    got = m.add_seq_tokens(next_id, prompt)
                    assert got % block_size == 0 and got <= (len(prompt) - 1) // block_size * block_size
                    texts[next_id] = prompt
                    next_id += 1
                continue
            if op == 5:
                if live:
                    m.swap_out([int(x) for x in rng.permutation(live)[:rng.integers(1, min(3, len(live)) + 1)]])
                continue
            if op == 6:
                if gone:
                    m.swap_in([int(x) for x in rng.permutation(gone)[:rng.integers(1, len(gone) + 1)]])
                continue
            if op == 7:
                p = prompts[rng.integers(len(prompts))]
                n = int(rng.integers(1, len(p) + 1))
                tail = list(rng.integers(0, 5, size=int(rng.integers(0, 3))))
                m.add_seq_tokens(next_id, p[:n] + tail)
                texts[next_id] = [int(t) for t in p[:n] + tail]
                next_id += 1
                continue
            if op == 0 or not live:
                shared = []
                if live and rng.random() < 0.5:
                    donor = live[rng.integers(len(live))]
                    full = m.lens[donor] // block_size
                    shared = m.tables[donor][:rng.integers(0, full + 1)]
                m.add_seq(next_id, len(shared) * block_size + int(rng.integers(0, 9)), shared)
                next_id += 1
            elif op == 1:
                parent = live[rng.integers(len(live))]
                m.fork(parent, next_id)
                texts[next_id] = None if texts.get(parent) is None else list(texts[parent])
                next_id += 1
            elif op == 2:
                pick = [int(s) for s in rng.permutation(live)[:rng.integers(1, len(live) + 1)]]
                m.append_slots(pick)
                for s_ in pick:
                    texts[s_] = None
            elif op == 3:
                every = sorted(m.tables)
                victim = every[rng.integers(len(every))]
                m.free_seq(victim)
                texts.pop(victim, None)
            else:
                s = live[rng.integers(len(live))]
                if m.lens[s]:
                    start = int(rng.integers(0, m.lens[s]))
                    m.slots(s, start, m.lens[s] - start)
        except BlockManagerError as e:
            assert e.code == ERR_OOM
        finally:
            check_invariants(m)
            check_histories(m, texts)
    return m


@pytest.mark.parametrize("seed", range(6))
def test_invariants_under_random_operations(seed):
    random_ops(seed)


def test_slots_follow_tables():
    m = random_ops(42, steps=200)
    for s, table in m.tables.items():
        got = m.slots(s, 0, m.lens[s])
        for p, slot in enumerate(got):
            assert slot // m.block_size == table[p // m.block_size]
            assert slot % m.block_size == p % m.block_size


@pytest.mark.parametrize("seed", range(6))
def test_invariants_under_random_operations_with_swap_and_prefix_cache(seed):
    m = random_ops(100 + seed, extended=True)
    assert m.num_cached_blocks() > 0


# ---------------------------------------------------------------------------
# Swap space
# ---------------------------------------------------------------------------

def test_swap_out_and_in_by_hand():
    m = BlockManagerModel(8, 4, list(range(8)), num_host_blocks=4)
    m.add_seq(0, 6)                    # device blocks 0, 1
    m.fork(0, 1)                       # shares 0, 1
    m.add_seq(2, 3)                    # block 2
    pairs = m.swap_out([0, 1])
    assert pairs == [(0, 0), (1, 1)]   # each distinct device block gets one host block
    assert m.tables[0] == m.tables[1] == [0, 1] and m.host_ref[:2] == [2, 2]
    assert m.num_free() == 7 and list(m.free) == [3, 4, 5, 6, 7, 0, 1]
    assert m.is_swapped(0) and not m.is_swapped(2)
    with pytest.raises(BlockManagerError) as e:
        m.append_slots([0])
    assert e.value.code == ERR_INVALID
    pairs = m.swap_in([1, 0])
    assert pairs == [(0, 3), (1, 4)]   # fresh device blocks from the front of the free list
    assert m.tables[0] == m.tables[1] == [3, 4] and m.ref[3] == m.ref[4] == 2
    assert m.num_host_free() == 4
    check_invariants(m)


def test_swap_partial_sharing_keeps_device_copy():
    """A block still used by a resident sequence stays on the device; the swapped
    sequence takes a host copy of it."""
    m = BlockManagerModel(6, 4, list(range(6)), num_host_blocks=3)
    m.add_seq(0, 8)                    # blocks 0, 1
    m.fork(0, 1)
    pairs = m.swap_out([1])
    assert pairs == [(0, 0), (1, 1)] and m.ref[0] == m.ref[1] == 1
    m.free_seq(1)                      # freeing a swapped-out sequence frees its host blocks
    assert m.num_host_free() == 3
    check_invariants(m)


def test_swap_is_all_or_nothing():
    m = BlockManagerModel(6, 4, list(range(6)), num_host_blocks=2)
    m.add_seq(0, 9)                    # 3 blocks > 2 host blocks
    with pytest.raises(BlockManagerError) as e:
        m.swap_out([0])
    assert e.value.code == ERR_OOM
    assert m.tables[0] == [0, 1, 2] and not m.is_swapped(0) and m.num_host_free() == 2
    m2 = BlockManagerModel(3, 4, list(range(3)), num_host_blocks=3)
    m2.add_seq(0, 8)
    m2.swap_out([0])
    m2.add_seq(1, 12)                  # takes every device block
    with pytest.raises(BlockManagerError) as e:
        m2.swap_in([0])
    assert e.value.code == ERR_OOM and m2.is_swapped(0)
    check_invariants(m2)


# ---------------------------------------------------------------------------
# Prefix caching
# ---------------------------------------------------------------------------

def test_fnv1a64_published_vectors():
    """FNV-1a 64-bit test vectors from the algorithm's published test suite."""
    assert fnv1a64(b"") == 0xCBF29CE484222325
    assert fnv1a64(b"a") == 0xAF63DC4C8601EC8C
    assert fnv1a64(b"foobar") == 0x85944171F73967E8


def test_block_hash_layout():
    """Parent hash as 8 little-endian bytes, then int32 little-endian token ids."""
    data = bytes([1, 0, 0, 0, 0, 0, 0, 0]) + bytes([7, 0, 0, 0]) + bytes([0xFF, 0xFF, 0xFF, 0xFF])
    assert block_hash(1, [7, -1]) == fnv1a64(data)


def test_prefix_cache_by_hand():
    bs = 4
    m = BlockManagerModel(12, bs, list(range(12)))
    a = list(range(100, 110))                         # 10 tokens: 2 full blocks + 2
    assert m.add_seq_tokens(0, a) == 0                # nothing cached yet
    assert m.tables[0] == [0, 1, 2] and m.num_cached_blocks() == 2
    b = a[:8] + [7, 7, 7]
    assert m.add_seq_tokens(1, b) == 8                # both full blocks shared
    assert m.tables[1][:2] == [0, 1] and m.ref[0] == m.ref[1] == 2
    c = a[:8]                                         # the last token sits in block 1:
    assert m.add_seq_tokens(2, c) == 4                # only block 0 is taken
    assert m.tables[2] == [0, 4] and m.num_cached_blocks() == 2   # block 4 holds a registered hash: not re-registered
    d = [5] + a[1:8]                                  # first block differs: no hit at all
    assert m.add_seq_tokens(3, d) == 0
    check_invariants(m)


def test_prefix_cache_revive_and_evict():
    bs = 4
    m = BlockManagerModel(8, bs, list(range(8)))
    p = list(range(12))
    m.add_seq_tokens(0, p + [99])                     # blocks 0,1,2 full (registered), 3 partial
    m.free_seq(0)                                     # all free again, 3 still registered
    assert m.num_free() == 8 and m.num_cached_blocks() == 3
    assert list(m.free) == [4, 5, 6, 7, 0, 1, 2, 3]
    assert m.add_seq_tokens(1, p + [98]) == 12        # revived from the free list
    assert m.tables[1] == [0, 1, 2, 4] and list(m.free) == [5, 6, 7, 3]
    m.free_seq(1)
    m.add_seq(2, 24)                                  # takes 5, 6, 7, 3, 0, 1: evicts 0 and 1
    assert m.tables[2] == [5, 6, 7, 3, 0, 1] and m.num_cached_blocks() == 1
    assert m.add_seq_tokens(3, p[:4] + [1]) == 0      # block 0's hash is gone
    assert m.tables[3] == [2, 4]                      # block 2 handed out: its old hash evicted,
    assert m.num_cached_blocks() == 1                 # the new prompt's first block registered
    check_invariants(m)


def test_prefix_cache_oom_is_all_or_nothing():
    m = BlockManagerModel(4, 4, list(range(4)))
    m.add_seq_tokens(0, list(range(9)))               # 3 blocks
    before = (list(m.free), list(m.ref), dict(m.cached))
    with pytest.raises(BlockManagerError) as e:
        m.add_seq_tokens(1, list(range(8)) + list(range(50, 60)))   # 2 cached + 3 fresh > 1 free
    assert e.value.code == ERR_OOM
    assert before == (list(m.free), list(m.ref), dict(m.cached)) and 1 not in m.tables


def decode_registration_example(m):
    """Hand-worked: 8 blocks of 4, free list 0..7.  Returns what the checks compare."""
    out = {}

    def table(seq, width):
        t, _ = m.export_tables([seq], width)
        return [int(x) for x in np.asarray(t)[0]]
    out["admit0"] = m.add_seq_tokens(0, [1, 2, 3, 4, 5, 6])   # block 0 full (registered), block 1 holds 5, 6
    out["cached0"] = m.num_cached_blocks()
    m.append_tokens([0], [7])
    out["cached1"] = m.num_cached_blocks()                      # block 1 not full yet
    slots, pairs = m.append_tokens([0], [8])                    # completes block 1
    out["slot8"] = [int(x) for x in slots]
    out["cached2"] = m.num_cached_blocks()
    out["admit1"] = m.add_seq_tokens(1, [1, 2, 3, 4, 5, 6, 7, 8, 9])   # continues the generated text
    out["table1"] = table(1, 3)
    m.append_slots([0])                                         # history of 0 ends here
    for t in (10, 11, 12):
        m.append_tokens([0], [t])                               # fills block 3 of seq 0: not registered
    out["cached3"] = m.num_cached_blocks()
    out["table0"] = table(0, 3)
    m.fork(1, 2)                                                # the child keeps 1's history
    _, pairs = m.append_tokens([1, 2], [10, 10])                # 1 copies its shared last block (2 -> 4)
    out["pairs"] = [tuple(int(v) for v in p) for p in pairs]
    m.append_tokens([1, 2], [11, 11])
    m.append_tokens([1, 2], [12, 12])                           # equal texts: 1 registers, 2 finds the hash taken
    out["cached4"] = m.num_cached_blocks()
    out["table1_after"], out["table2"] = table(1, 3), table(2, 3)
    return out


def test_decode_filled_blocks_register():
    m = BlockManagerModel(8, 4, list(range(8)))
    out = decode_registration_example(m)
    assert out["admit0"] == 0 and out["cached0"] == 1 and out["cached1"] == 1
    assert out["slot8"] == [1 * 4 + 3] and out["cached2"] == 2
    h0 = block_hash(0, [1, 2, 3, 4])
    h1 = block_hash(h0, [5, 6, 7, 8])
    assert m.cached[h0] == 0 and m.cached[h1] == 1
    assert out["admit1"] == 8 and out["table1"] == [0, 1, 2]
    assert out["cached3"] == 2 and out["table0"] == [0, 1, 3]
    assert out["pairs"] == [(2, 4)] and out["table1_after"] == [0, 1, 4] and out["table2"] == [0, 1, 2]
    h2 = block_hash(h1, [9, 10, 11, 12])
    assert out["cached4"] == 3 and m.cached[h2] == 4
    check_invariants(m)


@pytest.mark.parametrize("seed", range(4))
def test_decode_registration_under_random_operations(seed):
    random_ops(300 + seed, extended=True)
