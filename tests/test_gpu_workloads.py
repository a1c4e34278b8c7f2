"""Whole decode steps of the prefix-sharing / beam-fork workload and of the
long-context continuous-batching trace, driven by the C++ block manager and
checked against the oracle at every step.

Each step runs the full path: the host allocator hands out slots (and copy-on-write
pairs), copy_blocks copies the diverging shared blocks, reshape_and_cache writes the
new tokens, and paged_attention_decode attends over the tables.  The oracle side
replays the same operations with the reference allocator model and the oracle cache
ops on host arrays: tables, slots, pairs and the whole pool must match bit for bit,
attention within the stated tolerance.
"""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import cache_ops
from oracle import paged_attention as oracle
from oracle.block_manager import BlockManagerModel
from tests.gpu_helpers import compare, dev_bf16, host_bits

pytestmark = pytest.mark.gpu


class Lockstep:
    """The C++ block manager and the reference model, driven together."""

    def __init__(self, pkv, num_blocks, block_size, order):
        self.cpp = pkv.BlockManager(num_blocks, block_size, order)
        self.ref = BlockManagerModel(num_blocks, block_size, order)
        self.bs = block_size

    def add_seq(self, sid, n, shared=()):
        self.cpp.add_seq(sid, n, shared)
        self.ref.add_seq(sid, n, shared)

    def fork(self, parent, child):
        self.cpp.fork(parent, child)
        self.ref.fork(parent, child)

    def free_seq(self, sid):
        self.cpp.free_seq(sid)
        self.ref.free_seq(sid)

    def append(self, ids):
        slots, pairs = self.cpp.append_slots(ids)
        rslots, rpairs = self.ref.append_slots(ids)
        assert slots.tolist() == rslots and [tuple(p) for p in pairs.tolist()] == rpairs
        return slots, pairs

    def slots(self, sid, start, count):
        got = self.cpp.slots(sid, start, count)
        assert got.tolist() == self.ref.slots(sid, start, count)
        return got

    def tables(self, ids, max_blocks):
        t, l = self.cpp.export_tables(ids, max_blocks)
        rt, rl = self.ref.export_tables(ids, max_blocks)
        assert t.tolist() == rt and l.tolist() == rl
        assert self.cpp.num_free() == self.ref.num_free()
        return t, l


class Pool:
    """Device pool and its host mirror, written through the library and the oracle."""

    def __init__(self, pkv, rng, num_blocks, hkv, bs, d):
        self.pkv = pkv
        self.hkv, self.d = hkv, d
        self.k = wl.bf16_normal(rng, (num_blocks, hkv, bs, d))
        self.v = wl.bf16_normal(rng, (num_blocks, hkv, bs, d))
        self.dk, self.dv = dev_bf16(self.k), dev_bf16(self.v)
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def write(self, k, v, slots):
        self.pkv.reshape_and_cache(dev_bf16(k), dev_bf16(v), self.dk, self.dv,
                                   torch.from_numpy(np.asarray(slots, np.int64)).cuda(), status=self.status)
        self.k, self.v = cache_ops.reshape_and_cache(k, v, self.k, self.v, slots)

    def copy(self, pairs):
        if len(pairs) == 0:
            return
        self.pkv.copy_blocks([self.dk], [self.dv], torch.from_numpy(np.asarray(pairs, np.int64)).cuda(),
                             status=self.status)
        ks, vs = cache_ops.copy_blocks([self.k], [self.v], pairs)
        self.k, self.v = ks[0], vs[0]

    def check(self):
        torch.cuda.synchronize()
        assert self.status.item() == 0
        assert np.array_equal(host_bits(self.dk), self.k) and np.array_equal(host_bits(self.dv), self.v)


def decode_and_compare(pkv, pool, q_bits, tables, lens, scale, hq):
    ref = oracle.paged_decode(q_bits, pool.k, pool.v, tables, lens, scale)
    dq = dev_bf16(q_bits)
    dt, dl = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    maxl = int(lens.max())
    for path in (1, 2) if hq // pool.hkv > 1 else (1,):
        ws = torch.empty(pkv.paged_attention_workspace_size(len(lens), hq, pool.hkv, pool.d, pool.k.shape[2], maxl),
                         dtype=torch.uint8, device="cuda")
        out = torch.empty((len(lens), hq, pool.d), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        pkv.paged_attention_decode(out, dq, pool.dk, pool.dv, dt, dl, maxl, scale, ws, path=path, status=st)
        torch.cuda.synchronize()
        assert st.item() == 0
        compare(out.cpu().numpy(), ref)


def test_prefix_sharing_then_beam_fork(pkv):
    """The shared system prompt (one copy, referenced by every table) and 4-beam forks
    whose partially filled last block is copied on write (Outcome School vLLM
    explainer, "内存共享")."""
    rng = wl.rng_for(400)
    B, Hq, Hkv, D, bs = 12, 32, 8, 128, 16
    prefix_blocks = 16                      # a 256-token shared prompt
    suffix = rng.integers(10, 120, size=B)
    suffix[0] = 37                          # seq 0 owns the prompt's blocks
    lens = prefix_blocks * bs + suffix
    need = int(np.sum(-(-lens // bs))) - prefix_blocks * (B - 1) + 4 * B + 8 * B
    nb = int(need * 1.5)
    order = rng.permutation(nb).astype(np.int32)
    ls = Lockstep(pkv, nb, bs, order)
    pool = Pool(pkv, rng, nb, Hkv, bs, D)
    # the prompt is written once, through sequence 0
    ls.add_seq(0, int(lens[0]))
    prompt = ls.ref.tables[0][:prefix_blocks]
    for s in range(1, B):
        ls.add_seq(s, int(lens[s]), prompt)
    assert all(ls.cpp.refcount(b) == B for b in prompt)
    for s in range(B):
        start = 0 if s == 0 else prefix_blocks * bs
        slots = ls.slots(s, start, int(lens[s]) - start)
        k, v = wl.new_tokens(rng, len(slots), Hkv, D)
        pool.write(k, v, slots)
    pool.check()
    ids = list(range(B))
    max_blocks = int(np.max(-(-(lens + 8) // bs)))

    # phase A: one decode step over the sharing sequences
    slots, pairs = ls.append(ids)
    assert len(pairs) == 0
    k, v = wl.new_tokens(rng, B, Hkv, D)
    pool.write(k, v, slots)
    tables, clens = ls.tables(ids, max_blocks)
    q = wl.bf16_normal(rng, (B, Hq, D))
    decode_and_compare(pkv, pool, q, tables, clens, wl.fp32_scale(D), Hq)

    # phase B: every sequence forks into 4 beams; each beam appends its own token
    beams = []
    for s in range(B):
        beams.append(s)
        for j in range(1, 4):
            child = 1000 + 4 * s + j
            ls.fork(s, child)
            beams.append(child)
    for _ in range(3):
        slots, pairs = ls.append(beams)
        pool.copy(pairs)                    # copy-on-write before the new rows land
        k, v = wl.new_tokens(rng, len(beams), Hkv, D)
        pool.write(k, v, slots)
        pool.check()
        tables, clens = ls.tables(beams, max_blocks)
        q = wl.bf16_normal(rng, (len(beams), Hq, D))
        decode_and_compare(pkv, pool, q, tables, clens, wl.fp32_scale(D), Hq)
    # beams of one parent still share the prompt blocks and the full blocks before the fork
    assert all(ls.cpp.refcount(b) == 4 * B for b in prompt)


def test_continuous_batching_trace(pkv):
    """Long-context trace: each step appends one token per running sequence, decodes,
    frees finished sequences and admits seeded arrivals while the pool allows."""
    p = wl.TraceParams(max_batch=4, len_lo=300, len_hi=2500, budget_lo=1, budget_hi=12, steps=24,
                       num_blocks=1200)
    initial, arrivals = wl.trace_events(p, seed=500)
    rng = wl.rng_for(501)
    order = rng.permutation(p.num_blocks).astype(np.int32)
    ls = Lockstep(pkv, p.num_blocks, p.block_size, order)
    pool = Pool(pkv, rng, p.num_blocks, p.num_kv_heads, p.block_size, p.head_dim)
    running = {}                            # seq id -> remaining steps
    next_id = 0

    def admit(length, budget):
        nonlocal next_id
        need = -(-length // p.block_size)
        if need > ls.cpp.num_free():
            return False
        sid = next_id
        next_id += 1
        ls.add_seq(sid, length - 1)         # the prompt; its last token comes with the next step
        slots = ls.slots(sid, 0, length - 1)
        k, v = wl.new_tokens(rng, len(slots), p.num_kv_heads, p.head_dim)
        pool.write(k, v, slots)             # synthetic prefill
        running[sid] = budget
        return True

    for length, budget in initial:
        admit(length, budget)
    max_blocks = (p.len_hi + p.steps + p.block_size) // p.block_size + 1
    for step in range(p.steps):
        ids = sorted(running)
        if ids:
            slots, pairs = ls.append(ids)
            assert len(pairs) == 0
            k, v = wl.new_tokens(rng, len(ids), p.num_kv_heads, p.head_dim)
            pool.write(k, v, slots)
            tables, clens = ls.tables(ids, max_blocks)
            q = wl.bf16_normal(rng, (len(ids), p.num_heads, p.head_dim))
            decode_and_compare(pkv, pool, q, tables, clens, wl.fp32_scale(p.head_dim), p.num_heads)
            for sid in ids:
                running[sid] -= 1
                if running[sid] == 0:
                    ls.free_seq(sid)
                    del running[sid]
        for length, budget in arrivals[step]:
            if len(running) < p.max_batch:
                admit(length, budget)
    pool.check()
    assert next_id > len(initial)           # the trace admitted new requests


def test_preempt_by_swap_then_resume(pkv):
    """Sequences swapped out to pinned host blocks (intelliparadigm article §4.2:
    swap_space), their device blocks reused by new requests, then swapped back in:
    tables, pools and attention still match the oracle."""
    from oracle import cache_ops as co
    rng = wl.rng_for(900)
    Hq, Hkv, D, bs, nb, hb = 16, 4, 128, 16, 160, 96
    order = rng.permutation(nb).astype(np.int32)
    cpp = pkv.BlockManager(nb, bs, order, num_host_blocks=hb)
    model = BlockManagerModel(nb, bs, order, num_host_blocks=hb)
    ls = Lockstep.__new__(Lockstep)
    ls.cpp, ls.ref, ls.bs = cpp, model, bs
    pool = Pool(pkv, rng, nb, Hkv, bs, D)
    host_k = np.zeros((hb, Hkv, bs, D), np.uint16)
    host_v = np.zeros((hb, Hkv, bs, D), np.uint16)
    hk = torch.zeros((hb, Hkv, bs, D), dtype=torch.bfloat16).pin_memory()
    hv = torch.zeros((hb, Hkv, bs, D), dtype=torch.bfloat16).pin_memory()
    lens = rng.integers(40, 300, size=6)
    for s, L in enumerate(lens):
        ls.add_seq(s, int(L))
        slots = ls.slots(s, 0, int(L))
        k, v = wl.new_tokens(rng, len(slots), Hkv, D)
        pool.write(k, v, slots)
    ids = list(range(6))
    cpp.fork(2, 10)
    model.fork(2, 10)
    ids.append(10)
    max_blocks = 40
    tables, clens = ls.tables(ids, max_blocks)
    decode_and_compare(pkv, pool, wl.bf16_normal(rng, (len(ids), Hq, D)), tables, clens, wl.fp32_scale(D), Hq)

    # preempt 1, 2 and its fork 10 (they share blocks): one host copy of each block
    out_ids = [1, 2, 10]
    pairs = cpp.swap_out(out_ids)
    assert [tuple(p) for p in pairs.tolist()] == model.swap_out(out_ids)
    dp = torch.from_numpy(pairs).cuda()
    pkv.swap_blocks(pool.dk, hk, dp)
    pkv.swap_blocks(pool.dv, hv, dp)
    host_k = co.swap_blocks(pool.k, host_k, pairs)
    host_v = co.swap_blocks(pool.v, host_v, pairs)
    torch.cuda.synchronize()
    assert np.array_equal(hk.view(torch.int16).numpy().view(np.uint16), host_k)
    # new requests take the freed device blocks and overwrite them
    for s in (20, 21):
        L = int(rng.integers(200, 400))
        ls.add_seq(s, L)
        slots = ls.slots(s, 0, L)
        k, v = wl.new_tokens(rng, len(slots), Hkv, D)
        pool.write(k, v, slots)
    ls.free_seq(20)
    # resume
    pairs = cpp.swap_in(out_ids)
    assert [tuple(p) for p in pairs.tolist()] == model.swap_in(out_ids)
    dp = torch.from_numpy(pairs).cuda()
    pkv.swap_blocks(hk, pool.dk, dp)
    pkv.swap_blocks(hv, pool.dv, dp)
    pool.k = co.swap_blocks(host_k, pool.k, pairs)
    pool.v = co.swap_blocks(host_v, pool.v, pairs)
    pool.check()
    ids = [0, 1, 2, 3, 4, 5, 10, 21]
    slots, pairs = ls.append(ids)
    pool.copy(pairs)
    k, v = wl.new_tokens(rng, len(ids), Hkv, D)
    pool.write(k, v, slots)
    tables, clens = ls.tables(ids, max_blocks)
    decode_and_compare(pkv, pool, wl.bf16_normal(rng, (len(ids), Hq, D)), tables, clens, wl.fp32_scale(D), Hq)


def test_prefix_cached_admission(pkv):
    """Requests sharing a long system prompt (Outcome School explainer, "内存共享"):
    the second and later requests take the prompt's full blocks from the prefix cache,
    only their uncached tokens are written, and attention matches the oracle."""
    rng = wl.rng_for(910)
    Hq, Hkv, D, bs, nb = 32, 8, 128, 16, 400
    order = rng.permutation(nb).astype(np.int32)
    ls = Lockstep(pkv, nb, bs, order)
    pool = Pool(pkv, rng, nb, Hkv, bs, D)
    prompt = [int(t) for t in rng.integers(0, 32000, size=203)]           # 12 full blocks + 11
    pk, pv = wl.new_tokens(rng, len(prompt), Hkv, D)                      # its K/V, one copy
    ids = []
    for r in range(5):
        tail = [int(t) for t in rng.integers(0, 32000, size=int(rng.integers(1, 60)))]
        toks = prompt + tail
        got = ls.cpp.add_seq_tokens(r, toks)
        assert got == ls.ref.add_seq_tokens(r, toks)
        assert got == (0 if r == 0 else 12 * bs)
        slots = ls.slots(r, got, len(toks) - got)
        tk, tv = wl.new_tokens(rng, len(tail), Hkv, D)
        k = np.concatenate([pk[got:], tk])
        v = np.concatenate([pv[got:], tv])
        pool.write(k, v, slots)
        ids.append(r)
    pool.check()
    assert ls.cpp.num_cached_blocks() == ls.ref.num_cached_blocks() >= 12
    tables, clens = ls.tables(ids, 20)
    assert all(tables[r][:12].tolist() == tables[0][:12].tolist() for r in ids)
    decode_and_compare(pkv, pool, wl.bf16_normal(rng, (len(ids), Hq, D)), tables, clens, wl.fp32_scale(D), Hq)


def test_decode_filled_blocks_serve_a_continuation(pkv):
    """Blocks a sequence fills while decoding register in the prefix cache
    (append_tokens), so a later request whose prompt continues the generated text
    takes them from the cache, writes only its uncached tokens, and attends exactly
    as the oracle does over the same text."""
    rng = wl.rng_for(920)
    Hq, Hkv, D, bs, nb = 32, 8, 128, 16, 64
    order = rng.permutation(nb).astype(np.int32)
    ls = Lockstep(pkv, nb, bs, order)
    pool = Pool(pkv, rng, nb, Hkv, bs, D)
    prompt = [int(t) for t in rng.integers(0, 32000, size=40)]    # blocks 0, 1 full; 32..39 in block 2
    gen = [int(t) for t in rng.integers(0, 32000, size=45)]       # positions 40..84: blocks 2, 3, 4 complete
    text = prompt + gen
    tk, tv = wl.new_tokens(rng, len(text), Hkv, D)                  # K/V of every position of the text
    assert ls.cpp.add_seq_tokens(0, prompt) == ls.ref.add_seq_tokens(0, prompt) == 0
    pool.write(tk[:40], tv[:40], ls.slots(0, 0, 40))
    for i, tok in enumerate(gen):
        slots, pairs = ls.cpp.append_tokens([0], [tok])
        rslots, rpairs = ls.ref.append_tokens([0], [tok])
        assert slots.tolist() == rslots and len(pairs) == len(rpairs) == 0
        pool.write(tk[40 + i:41 + i], tv[40 + i:41 + i], slots)
    assert ls.cpp.num_cached_blocks() == ls.ref.num_cached_blocks() == 5
    tail = [int(t) for t in rng.integers(0, 32000, size=7)]
    toks = text + tail                                              # 92 tokens
    got = ls.cpp.add_seq_tokens(1, toks)
    assert got == ls.ref.add_seq_tokens(1, toks) == 5 * bs          # every full block of the text
    nk, nv = wl.new_tokens(rng, len(tail), Hkv, D)
    pool.write(np.concatenate([tk[got:], nk]), np.concatenate([tv[got:], nv]), ls.slots(1, got, len(toks) - got))
    pool.check()
    tables, clens = ls.tables([0, 1], 6)
    assert tables[1][:5].tolist() == tables[0][:5].tolist() and tables[1][5] != tables[0][5]
    assert clens.tolist() == [len(text), len(toks)]
    decode_and_compare(pkv, pool, wl.bf16_normal(rng, (2, Hq, D)), tables, clens, wl.fp32_scale(D), Hq)
