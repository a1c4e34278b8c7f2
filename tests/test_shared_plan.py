"""Host planner of the shared-prefix decode (pkv_shared_plan), on the CPU.

The plan must (1) find exactly the segments the definition gives -- maximal runs of
whole blocks that a range of adjacent rows holds at the same table positions, nested
-- checked against a plain recursive restatement on batches built by the allocator
model (shared prompts, beam forks, appends that copy-on-write); (2) be a valid
decomposition: every part's rows really hold the part's blocks, full; every row's
shared parts tile its tokens [0, k*block_size) exactly once and its remainder is the
rest; every (part, row) is in exactly one work entry and has one partial id.
"""
import numpy as np
import pytest

import workloads as wl
from oracle.block_manager import BlockManagerModel


def reference_segments(tables, lens, bs, min_rows):
    """Segments (row0, nrows, block0, nblocks) and each row's private start, from the definition."""
    B, mb = tables.shape

    def full(r, k):
        return k < mb and (k + 1) * bs <= lens[r]

    segs, depth = [], [0] * B

    def split(r0, r1, k):
        r = r0
        while r < r1:
            if not full(r, k):
                r += 1
                continue
            s = r + 1
            while s < r1 and full(s, k) and tables[s][k] == tables[r][k]:
                s += 1
            if s - r >= min_rows:
                k2 = k + 1
                while all(full(q, k2) and tables[q][k2] == tables[r][k2] for q in range(r, s)):
                    k2 += 1
                segs.append((r, s - r, k, k2 - k))
                for q in range(r, s):
                    depth[q] = k2
                split(r, s, k2)
            r = s

    split(0, B, 0)
    return sorted(segs), depth


def decode_plan(plan, info):
    i = info

    def arr(off, n, w=1):
        return np.frombuffer(plan, np.int32, count=n * w, offset=int(off)).reshape(n, w) if n else np.zeros((0, w), np.int32)

    entries = arr(i.off_entries, i.num_entries, 4)
    parts = arr(i.off_parts, i.num_parts, 8)
    suffix = arr(i.off_suffix_lens, i.num_seqs)[:, 0]
    offset = arr(i.off_block_offset, i.num_seqs)[:, 0]
    row_start = arr(i.off_row_start, i.num_seqs + 1)[:, 0]
    row_ids = arr(i.off_row_ids, i.num_partials)[:, 0]
    return entries, parts, suffix, offset, row_start, row_ids


def check_plan(tables, lens, bs, g, plan, info, min_rows=2):
    B = len(lens)
    entries, parts, suffix, offset, row_start, row_ids = decode_plan(plan, info)
    segs, depth = reference_segments(tables, lens, bs, min_rows)
    assert info.num_segments == len(segs)
    assert offset.tolist() == depth
    assert suffix.tolist() == [int(lens[r]) - depth[r] * bs for r in range(B)]
    # every part: its rows hold its blocks, full
    got_segs = set()
    id_of = {}
    scratch = 0
    for p, (trow, blk0, nkeys, row0, nrows, first, base, z1) in enumerate(parts.tolist()):
        assert z1 == 0 and trow == row0 and 1 <= nkeys <= info.key_chunk and nkeys % bs == 0
        assert base == scratch  # scratch blocks of the 8-bit run, consecutive in plan order
        scratch += nkeys // bs
        nblk = nkeys // bs
        for r in range(row0, row0 + nrows):
            for k in range(blk0, blk0 + nblk):
                assert tables[r][k] == tables[trow][k] and (k + 1) * bs <= lens[r]
            id_of[(p, r)] = first + r - row0
        got_segs.add((row0, nrows))
    assert got_segs == {(s[0], s[1]) for s in segs}
    assert sorted(id_of.values()) == list(range(info.num_partials))
    # every row: its parts tile [0, depth * bs) exactly once, listed in its CSR row
    ids_to_part = {v: k for k, v in id_of.items()}
    for r in range(B):
        ids = row_ids[row_start[r]:row_start[r + 1]].tolist()
        covered = []
        for i in ids:
            p, rr = ids_to_part[i]
            assert rr == r
            blk0, nkeys = parts[p][1], parts[p][2]
            covered += list(range(blk0 * bs, blk0 * bs + nkeys))
        assert sorted(covered) == list(range(depth[r] * bs)), r
    assert row_start[0] == 0 and row_start[-1] == info.num_partials
    # entries: each (part, row) once; tiles of at most 128 / g rows; tile B only after a full tile A
    tile = 128 // g
    seen = []
    for x, y, z, p in entries.tolist():
        na, nb = z & 0xFF, (z >> 8) & 0xFF
        assert y == 0 and z >> 16 == 0 and 1 <= na <= tile and nb <= tile and (nb == 0 or na == tile)
        row0, nrows = parts[p][3], parts[p][4]
        assert row0 <= x and x + na + nb <= row0 + nrows
        seen += [(p, r) for r in range(x, x + na + nb)]
    assert sorted(seen) == sorted(id_of)
    # parts with more keys come first
    nk = [parts[entries[e][3]][2] for e in range(len(entries))]
    assert nk == sorted(nk, reverse=True)
    assert info.shared_row_tokens == sum(depth) * bs
    assert scratch * bs == info.shared_tokens


def beam_batch(seed, parents=6, beams=4, prompt_blocks=3, bs=16, steps=2):
    """A prompt shared by every parent, each parent forked into beams (adjacent rows),
    then `steps` appended tokens (the first copies shared partial last blocks)."""
    rng = wl.rng_for(seed)
    nb = 400
    m = BlockManagerModel(nb, bs, initial_order=rng.permutation(nb).astype(np.int32))
    lens = prompt_blocks * bs + rng.integers(0, 70, size=parents)
    m.add_seq(0, int(lens[0]))
    prefix = m.tables[0][:prompt_blocks]
    for s in range(1, parents):
        m.add_seq(s, int(lens[s]), prefix)
    ids = []
    for s in range(parents):
        ids.append(s)
        for k in range(beams - 1):
            c = parents + s * (beams - 1) + k
            m.fork(s, c)
            ids.append(c)
    for _ in range(steps):
        m.append_slots(ids)
    mb = max(len(m.tables[i]) for i in ids) + 2
    t, l = m.export_tables(ids, mb)
    return np.asarray(t, np.int32), np.asarray(l, np.int32), bs


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("steps", [0, 1, 5])
def test_plan_of_beam_batches(pkv, seed, steps):
    tables, lens, bs = beam_batch(seed, steps=steps)
    for g in (4, 8):
        plan, info = pkv.shared_plan(tables, lens, 8 * g, 8, bs)
        check_plan(tables, lens, bs, g, plan.tobytes(), info)


@pytest.mark.parametrize("seed", range(4))
def test_plan_of_random_sharing(pkv, seed):
    """Rows copy runs of other rows' tables at random (shared or not), lengths cut
    anywhere (partial blocks are never shared); the plan matches the definition."""
    rng = wl.rng_for(100 + seed)
    B, mb, bs = 40, 12, 16
    tables = rng.integers(0, 50, size=(B, mb)).astype(np.int32)
    for r in range(1, B):
        if rng.random() < 0.7:
            k = int(rng.integers(0, mb + 1))
            tables[r, :k] = tables[r - 1, :k]
    lens = rng.integers(0, mb * bs + 1, size=B).astype(np.int32)
    for min_rows in (2, 3):
        plan, info = pkv.shared_plan(tables, lens, 16, 4, bs, min_rows=min_rows)
        check_plan(tables, lens, bs, 4, plan.tobytes(), info, min_rows)


def test_plan_of_the_shared_prompt_batch(pkv):
    """The shared-prefix workload: one segment of all 128 rows over the 64 prompt blocks;
    with 4 beams, that segment over 512 rows plus one per parent over its full suffix blocks."""
    b = wl.make_decode_batch("prefix_beams", with_data=False)
    import bench
    lens = b.context_lens.astype(np.int64)
    nb = int(np.ceil(1.3 * np.sum(-(-(lens + 8) // 16)) * 4))
    order = wl.rng_for(7).permutation(nb).astype(np.int32)
    mb = int(np.max(-(-(lens + 8) // 16)))
    bm = bench.build_manager(pkv.BlockManager, nb, 16, order, lens, wl.PREFIX_TOKENS // 16, mb)
    tables, l = bm.export_tables(range(b.num_seqs), mb)
    plan, info = pkv.shared_plan(tables, l, 32, 8, 16)
    assert info.num_segments == 1 and info.shared_tokens == wl.PREFIX_TOKENS
    check_plan(tables, l, 16, 4, plan.tobytes(), info)
    bm.close()
    bm = bench.build_manager(pkv.BlockManager, nb, 16, order, lens, wl.PREFIX_TOKENS // 16, mb, 4)
    ids = bench.beam_ids(b.num_seqs, 4)
    bm.append_slots(ids)
    tables, l = bm.export_tables(ids, mb)
    plan, info = pkv.shared_plan(tables, l, 32, 8, 16)
    full_suffix = (lens - wl.PREFIX_TOKENS) // 16          # parents' full private blocks before the append
    assert info.num_segments == 1 + int(np.sum(full_suffix > 0))
    check_plan(tables, l, 16, 4, plan.tobytes(), info)
    bm.close()


def test_key_chunks(pkv):
    tables, lens, bs = beam_batch(3, parents=4, beams=2, prompt_blocks=40, steps=0)
    for chunk in (128, 256, 1024):
        plan, info = pkv.shared_plan(tables, lens, 16, 4, bs, key_chunk=chunk)
        assert info.key_chunk == chunk
        check_plan(tables, lens, bs, 4, plan.tobytes(), info)
    plan, info = pkv.shared_plan(tables, lens, 16, 4, bs)       # automatic: small batch, short chunks
    assert info.key_chunk == 128


def test_no_sharing_and_empty_rows(pkv):
    tables = np.arange(24, dtype=np.int32).reshape(4, 6)
    lens = np.array([0, 96, 17, 5], np.int32)
    plan, info = pkv.shared_plan(tables, lens, 8, 2, 16)
    assert info.num_segments == info.num_entries == info.num_partials == 0
    check_plan(tables, lens, 16, 4, plan.tobytes(), info)
    plan, info = pkv.shared_plan(np.zeros((0, 4), np.int32), np.zeros(0, np.int32), 8, 2, 16)
    assert info.num_seqs == 0


def test_plan_errors(pkv):
    t = np.zeros((2, 4), np.int32)
    with pytest.raises(pkv.PkvError) as e:
        pkv.shared_plan(t, np.array([0, 65], np.int32), 8, 2, 16)         # longer than the table
    assert e.value.code == pkv.PKV_ERR_INVALID
    with pytest.raises(pkv.PkvError) as e:
        pkv.shared_plan(t, np.array([0, 16], np.int32), 8, 2, 16, min_rows=1)
    assert e.value.code == pkv.PKV_ERR_INVALID
    with pytest.raises(pkv.PkvError) as e:
        pkv.shared_plan(t, np.array([0, 16], np.int32), 8, 2, 16, key_chunk=100)
    assert e.value.code == pkv.PKV_ERR_INVALID
    with pytest.raises(pkv.PkvError) as e:
        pkv.shared_plan(t, np.array([0, 16], np.int32), 6, 2, 16)          # group 3 does not divide 128
    assert e.value.code == pkv.PKV_ERR_UNSUPPORTED
    import ctypes
    info = pkv.SharedPlanInfo()
    lens = np.array([16, 16], np.int32)
    lib = pkv.library()
    assert lib.pkv_shared_plan(t.ctypes.data, 4, lens.ctypes.data, 2, 8, 2, 16, 2, 0, None, 0, ctypes.byref(info)) == 0
    small = np.zeros(max(int(info.bytes) - 16, 0), np.uint8)
    assert lib.pkv_shared_plan(t.ctypes.data, 4, lens.ctypes.data, 2, 8, 2, 16, 2, 0, small.ctypes.data, small.nbytes,
                               ctypes.byref(info)) == pkv.PKV_ERR_INVALID


def test_workspace_size_of_the_shared_run(pkv):
    tables, lens, bs = beam_batch(1)
    plan, info = pkv.shared_plan(tables, lens, 32, 8, bs)
    n = pkv.paged_attention_decode_shared_workspace_size(info, 32, 8, 128)
    assert n >= info.num_partials * 32 * (128 * 4 + 8)
    assert pkv.paged_attention_decode_shared_workspace_size(info, 32, 8, 64) == 0


def test_plan_into_a_caller_buffer(pkv):
    """One call into a caller-provided buffer gives the same plan; a short buffer raises."""
    tables, lens, bs = beam_batch(2)
    plan, info = pkv.shared_plan(tables, lens, 32, 8, bs)
    buf = np.full(plan.nbytes + 100, 0xAB, np.uint8)
    got, info2 = pkv.shared_plan(tables, lens, 32, 8, bs, out=buf)
    assert got.nbytes == plan.nbytes and np.array_equal(got, plan) and info2.as_dict() == info.as_dict()
    with pytest.raises(pkv.PkvError):
        pkv.shared_plan(tables, lens, 32, 8, bs, out=np.zeros(plan.nbytes - 16, np.uint8))
