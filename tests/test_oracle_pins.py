"""Pins for the attention and cache-op oracle (CPU only).

Each check ties the oracle to something other than itself: a closed form, a
library attention routine (torch scaled_dot_product_attention in float64), an
invariant the pages state, or an explicit element loop on a tiny input.  The
mutation tests at the end plant plausible mistakes in copies of the oracle's
source and require that at least one pin catches each.
"""
import inspect
import math
import textwrap

import numpy as np
import pytest
import torch

import workloads as wl
from oracle import cache_ops, paged_attention

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


# ---------------------------------------------------------------------------
# Test-side construction of paged storage from contiguous per-sequence data.
# Token t of a sequence lives in logical block t // bs at row t % bs, and the
# table maps logical block -> physical block (vLLM 初探 §1.4 figure).
# ---------------------------------------------------------------------------

def scatter_to_pool(contig_bits, lens, tables, num_blocks, block_size):
    """contig_bits [B, Hkv, max_len, D] -> pool [NB, Hkv, bs, D] (unused rows random)."""
    B, Hkv, _, D = contig_bits.shape
    rng = wl.rng_for(99)
    pool = wl.bf16_normal(rng, (num_blocks, Hkv, block_size, D))
    for s in range(B):
        for t in range(int(lens[s])):
            blk = tables[s][t // block_size]
            pool[blk, :, t % block_size, :] = contig_bits[s, :, t, :]
    return pool


def random_case(seed, B=3, Hq=4, Hkv=2, D=16, bs=4, max_len=13, lens=None):
    rng = wl.rng_for(seed)
    if lens is None:
        lens = rng.integers(1, max_len + 1, size=B).astype(np.int32)
    lens = np.asarray(lens, np.int32)
    need = -(-lens // bs)
    nb = int(need.sum()) + 5
    order = rng.permutation(nb).astype(np.int32)
    tables = wl.place_blocks(lens, bs, order)
    L = int(lens.max())
    q = wl.bf16_normal(rng, (B, Hq, D))
    k = wl.bf16_normal(rng, (B, Hkv, L, D))
    v = wl.bf16_normal(rng, (B, Hkv, L, D))
    kc = scatter_to_pool(k, lens, tables, nb, bs)
    vc = scatter_to_pool(v, lens, tables, nb, bs)
    return dict(q=q, k=k, v=v, kc=kc, vc=vc, tables=tables, lens=lens, nb=nb, bs=bs,
                scale=wl.fp32_scale(D), order=order)


def f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sdpa_reference(q_bits, k_bits, v_bits, lens, scale):
    """torch's scaled_dot_product_attention in float64 on contiguous K/V."""
    B, Hq, D = q_bits.shape
    Hkv = k_bits.shape[1]
    out = np.zeros((B, Hq, D))
    for s in range(B):
        L = int(lens[s])
        if L == 0:
            continue
        q = torch.from_numpy(f64(q_bits[s]))[:, None, :]               # [Hq, 1, D]
        k = torch.from_numpy(f64(k_bits[s, :, :L])).repeat_interleave(Hq // Hkv, 0)
        v = torch.from_numpy(f64(v_bits[s, :, :L])).repeat_interleave(Hq // Hkv, 0)
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=float(np.float32(scale)))
        out[s] = o[:, 0, :].numpy()
    return out


# ---------------------------------------------------------------------------
# Pins as functions of an implementation, so mutants can be run through them.
# ---------------------------------------------------------------------------

def pin_library_attention(impl):
    for seed in range(4):
        c = random_case(seed)
        got = impl(c["q"], c["kc"], c["vc"], c["tables"], c["lens"], c["scale"])
        ref = sdpa_reference(c["q"], c["k"], c["v"], c["lens"], c["scale"])
        if not np.allclose(got, ref, rtol=0, atol=1e-12):
            return False
    return True


def pin_single_token(impl):
    c = random_case(11, lens=[1, 1, 1])
    got = impl(c["q"], c["kc"], c["vc"], c["tables"], c["lens"], c["scale"])
    g = got.shape[1] // c["kc"].shape[1]
    for s in range(3):
        for h in range(got.shape[1]):
            expect = f64(c["vc"][c["tables"][s][0], h // g, 0])
            if not np.array_equal(got[s, h], expect):
                return False
    return True


def pin_constant_keys_mean(impl):
    c = random_case(12, lens=[5, 9, 13])
    k_const = c["k"].copy()
    k_const[:] = c["k"][:, :, :1, :]          # every key of a sequence/head equals its first key
    kc = scatter_to_pool(k_const, c["lens"], c["tables"], c["nb"], c["bs"])
    got = impl(c["q"], kc, c["vc"], c["tables"], c["lens"], c["scale"])
    g = got.shape[1] // kc.shape[1]
    for s in range(3):
        L = int(c["lens"][s])
        for h in range(got.shape[1]):
            expect = f64(c["v"][s, h // g, :L]).mean(axis=0)
            if not np.allclose(got[s, h], expect, rtol=0, atol=1e-13):
                return False
    return True


def pin_scale_zero_mean(impl):
    c = random_case(13, lens=[3, 8, 11])
    got = impl(c["q"], c["kc"], c["vc"], c["tables"], c["lens"], 0.0)
    g = got.shape[1] // c["kc"].shape[1]
    for s in range(3):
        L = int(c["lens"][s])
        for h in range(got.shape[1]):
            if not np.allclose(got[s, h], f64(c["v"][s, h // g, :L]).mean(axis=0), rtol=0, atol=1e-13):
                return False
    return True


def pin_dominant_key(impl):
    """One key aligned with a large query dominates: output ~= its value row."""
    c = random_case(14, lens=[10, 10, 10], D=16)
    q = np.zeros_like(c["q"])
    q[:] = wl.f32_to_bf16_bits(np.full(q.shape, 8.0, np.float32))
    k = np.zeros_like(c["k"])                  # zero keys ...
    star = 6
    k[:, :, star, :] = wl.f32_to_bf16_bits(np.full((16,), 8.0, np.float32))  # ... except token 6
    kc = scatter_to_pool(k, c["lens"], c["tables"], c["nb"], c["bs"])
    got = impl(q, kc, c["vc"], c["tables"], c["lens"], 1.0)
    g = got.shape[1] // kc.shape[1]
    for s in range(3):
        for h in range(got.shape[1]):
            if not np.allclose(got[s, h], f64(c["v"][s, h // g, star]), rtol=0, atol=1e-9):
                return False
    return True


def pin_block_permutation(impl):
    c = random_case(15, B=4, max_len=21)
    base = impl(c["q"], c["kc"], c["vc"], c["tables"], c["lens"], c["scale"])
    perm = wl.rng_for(7).permutation(c["nb"])
    kc2 = np.empty_like(c["kc"])
    vc2 = np.empty_like(c["vc"])
    kc2[perm] = c["kc"]
    vc2[perm] = c["vc"]
    tables2 = perm[c["tables"]].astype(np.int32)
    got = impl(c["q"], kc2, vc2, tables2, c["lens"], c["scale"])
    return np.array_equal(base, got)


def pin_block_size(impl):
    lens = np.array([1, 16, 17, 40, 64], np.int32)
    outs = []
    for bs in (16, 32):
        rng = wl.rng_for(16)
        B, Hq, Hkv, D = 5, 4, 2, 8
        q = wl.bf16_normal(rng, (B, Hq, D))
        k = wl.bf16_normal(rng, (B, Hkv, 64, D))
        v = wl.bf16_normal(rng, (B, Hkv, 64, D))
        nb = int((-(-lens // bs)).sum()) + 2
        tables = wl.place_blocks(lens, bs, wl.rng_for(bs).permutation(nb).astype(np.int32))
        kc = scatter_to_pool(k, lens, tables, nb, bs)
        vc = scatter_to_pool(v, lens, tables, nb, bs)
        outs.append(impl(q, kc, vc, tables, lens, 0.35))
    return np.allclose(outs[0], outs[1], rtol=0, atol=1e-12)


def pin_shared_prefix(impl):
    """Tables sharing prefix blocks == the same sequences with private copies."""
    rng = wl.rng_for(17)
    bs, Hkv, Hq, D = 4, 2, 4, 8
    prefix_blocks, B = 3, 4
    suffix = np.array([1, 4, 5, 7], np.int32)
    lens = prefix_blocks * bs + suffix
    nb_shared = prefix_blocks + int((-(-suffix // bs)).sum())
    q = wl.bf16_normal(rng, (B, Hq, D))
    order = rng.permutation(nb_shared + 20).astype(np.int32)
    tables_shared = wl.place_blocks(lens, bs, order, shared_prefix_blocks=prefix_blocks)
    kc = wl.bf16_normal(rng, (nb_shared + 20, Hkv, bs, D))
    vc = wl.bf16_normal(rng, (nb_shared + 20, Hkv, bs, D))
    # private copies of the prefix blocks for sequences 1..B-1
    nb_dup = nb_shared + 20 + prefix_blocks * (B - 1)
    kc_dup = np.concatenate([kc, np.zeros((nb_dup - kc.shape[0],) + kc.shape[1:], np.uint16)])
    vc_dup = np.concatenate([vc, np.zeros((nb_dup - vc.shape[0],) + vc.shape[1:], np.uint16)])
    tables_dup = tables_shared.copy()
    nxt = nb_shared + 20
    for s in range(1, B):
        for j in range(prefix_blocks):
            src = tables_shared[s][j]
            kc_dup[nxt] = kc[src]
            vc_dup[nxt] = vc[src]
            tables_dup[s][j] = nxt
            nxt += 1
    a = impl(q, kc, vc, tables_shared, lens, 0.3)
    b = impl(q, kc_dup, vc_dup, tables_dup, lens, 0.3)
    return np.array_equal(a, b)


def pin_gqa_repeat(impl):
    c = random_case(18, Hq=6, Hkv=2)
    gqa = impl(c["q"], c["kc"], c["vc"], c["tables"], c["lens"], c["scale"])
    kc_rep = np.repeat(c["kc"], 3, axis=1)
    vc_rep = np.repeat(c["vc"], 3, axis=1)
    mha = impl(c["q"], kc_rep, vc_rep, c["tables"], c["lens"], c["scale"])
    return np.array_equal(gqa, mha)


def pin_linearity(impl):
    rng = wl.rng_for(19)
    c = random_case(19)
    shape = c["vc"].shape
    v1 = wl.f32_to_bf16_bits(rng.integers(-4, 5, size=shape).astype(np.float32) / 4)
    v2 = wl.f32_to_bf16_bits(rng.integers(-4, 5, size=shape).astype(np.float32) / 4)
    vsum = wl.f32_to_bf16_bits(f64(v1).astype(np.float32) + f64(v2).astype(np.float32))
    o1 = impl(c["q"], c["kc"], v1, c["tables"], c["lens"], c["scale"])
    o2 = impl(c["q"], c["kc"], v2, c["tables"], c["lens"], c["scale"])
    o12 = impl(c["q"], c["kc"], vsum, c["tables"], c["lens"], c["scale"])
    return np.allclose(o12, o1 + o2, rtol=0, atol=1e-12)


def pin_zero_length(impl):
    c = random_case(20, lens=[0, 5, 0])
    got = impl(c["q"], c["kc"], c["vc"], c["tables"], c["lens"], c["scale"])
    return np.all(got[0] == 0) and np.all(got[2] == 0) and np.any(got[1] != 0)


ATTENTION_PINS = [pin_library_attention, pin_single_token, pin_constant_keys_mean, pin_scale_zero_mean,
                  pin_dominant_key, pin_block_permutation, pin_block_size, pin_shared_prefix,
                  pin_gqa_repeat, pin_linearity, pin_zero_length]


@pytest.mark.parametrize("pin", ATTENTION_PINS, ids=lambda p: p.__name__)
def test_attention_oracle_pin(pin):
    assert pin(paged_attention.paged_decode)


def test_paged_equals_contiguous_layout():
    """vLLM 初探 §1.4: the traditional layout is one contiguous [heads, seq_len, head_dim]
    slab per request; paging changes where K/V live, not the result (Outcome School
    explainer: vLLM does not change output quality)."""
    c = random_case(21, B=5, max_len=30)
    paged = paged_attention.paged_decode(c["q"], c["kc"], c["vc"], c["tables"], c["lens"], c["scale"])
    contig = paged_attention.contiguous_decode(c["q"], c["k"], c["v"], c["lens"], c["scale"])
    assert np.array_equal(paged, contig)


@pytest.mark.parametrize("prompt_len", [10, 12, 13])
def test_beam_fork_copy_on_write_gives_each_beam_its_own_sequence(prompt_len):
    """Outcome School explainer, "内存共享": beams share blocks until they diverge.  A
    prompt forked into 4 beams, each appending its own tokens (allocator model -> copy of
    the shared partial block -> cache write -> gather through the tables), must give
    every beam the attention of its own contiguous sequence (the prompt, then its own
    tokens); no beam's write may reach another beam.  Prompt lengths 10 and 13 leave a
    partial last block (three copies on the first append), 12 ends on a boundary."""
    from oracle.block_manager import BlockManagerModel
    rng = wl.rng_for(400 + prompt_len)
    bs, Hkv, Hq, D, beams, nb = 4, 2, 4, 8, 4, 40
    scale = wl.fp32_scale(D)
    m = BlockManagerModel(nb, bs, initial_order=rng.permutation(nb).astype(np.int32))
    m.add_seq(0, prompt_len)
    for b in range(1, beams):
        m.fork(0, b)
    ids = list(range(beams))
    kc = wl.bf16_normal(rng, (nb, Hkv, bs, D))
    vc = wl.bf16_normal(rng, (nb, Hkv, bs, D))
    pk = wl.bf16_normal(rng, (prompt_len, Hkv, D))
    pv = wl.bf16_normal(rng, (prompt_len, Hkv, D))
    kc, vc = cache_ops.reshape_and_cache(pk, pv, kc, vc, np.asarray(m.slots(0, 0, prompt_len), np.int64))
    own_k = [[pk[t] for t in range(prompt_len)] for _ in range(beams)]
    own_v = [[pv[t] for t in range(prompt_len)] for _ in range(beams)]
    for step in range(5):
        slots, pairs = m.append_slots(ids)
        if step == 0:
            assert len(pairs) == (0 if prompt_len % bs == 0 else beams - 1)
        if len(pairs):
            ks, vs = cache_ops.copy_blocks([kc], [vc], np.asarray(pairs, np.int64))
            kc, vc = ks[0], vs[0]
        nk = wl.bf16_normal(rng, (beams, Hkv, D))
        nv = wl.bf16_normal(rng, (beams, Hkv, D))
        kc, vc = cache_ops.reshape_and_cache(nk, nv, kc, vc, np.asarray(slots, np.int64))
        for b in range(beams):
            own_k[b].append(nk[b])
            own_v[b].append(nv[b])
        q = wl.bf16_normal(rng, (beams, Hq, D))
        tables, lens = m.export_tables(ids, 8)
        got = paged_attention.paged_decode(q, kc, vc, np.asarray(tables, np.int32), np.asarray(lens, np.int32), scale)
        L = prompt_len + step + 1
        ck = np.stack([np.stack(own_k[b], axis=1) for b in range(beams)])   # [beams, Hkv, L, D]
        cv = np.stack([np.stack(own_v[b], axis=1) for b in range(beams)])
        exp = paged_attention.contiguous_decode(q, ck, cv, np.full(beams, L, np.int32), scale)
        assert np.array_equal(got, exp)


def test_golden_block_table_figure_gather():
    """The figure's request A (Block 0 -> 3, Block 1 -> 7): positions 0..31 are read
    from physical blocks 3 then 7, in that order."""
    import json, os
    fig = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "block_table_figure.json")))
    table = fig["expected"]["table_A"]
    bs = fig["scenario"]["block_size"]
    pool = np.zeros((8, 1, bs, 1), np.uint16)
    for b in range(8):
        for r in range(bs):
            pool[b, 0, r, 0] = wl.f32_to_bf16_bits(np.array([b * 16 + r], np.float32))[0]
    got = paged_attention.gather_sequence(pool, np.array(table), 32)[:, 0, 0]
    expect = [3 * 16 + r for r in range(16)] + [7 * 16 + r for r in range(16)]
    assert got.tolist() == expect


# ---------------------------------------------------------------------------
# Cache ops: explicit element loops on tiny inputs
# ---------------------------------------------------------------------------

def test_reshape_and_cache_matches_element_loop():
    rng = wl.rng_for(30)
    NB, Hkv, bs, D, T = 6, 2, 4, 3, 7
    kc = wl.bf16_normal(rng, (NB, Hkv, bs, D))
    vc = wl.bf16_normal(rng, (NB, Hkv, bs, D))
    k = wl.bf16_normal(rng, (T, Hkv, D))
    v = wl.bf16_normal(rng, (T, Hkv, D))
    slots = np.array([0, 5, -1, 23, 9, -7, 14], np.int64)
    got_k, got_v = cache_ops.reshape_and_cache(k, v, kc, vc, slots)
    exp_k, exp_v = kc.copy(), vc.copy()
    for t in range(T):
        if slots[t] < 0:
            continue
        for h in range(Hkv):
            for d in range(D):
                exp_k[slots[t] // bs, h, slots[t] % bs, d] = k[t, h, d]
                exp_v[slots[t] // bs, h, slots[t] % bs, d] = v[t, h, d]
    assert np.array_equal(got_k, exp_k) and np.array_equal(got_v, exp_v)
    # rows of skipped tokens and untouched slots keep their old contents
    written = {int(s) for s in slots if s >= 0}
    for slot in range(NB * bs):
        if slot not in written:
            assert np.array_equal(got_k[slot // bs, :, slot % bs], kc[slot // bs, :, slot % bs])


def test_copy_blocks_parallel_semantics():
    rng = wl.rng_for(31)
    layers = [(wl.bf16_normal(rng, (5, 2, 4, 3)), wl.bf16_normal(rng, (5, 2, 4, 3))) for _ in range(2)]
    pairs = np.array([[0, 3], [3, 4]], np.int64)   # 3 is both a dst and (later) a src
    ks, vs = cache_ops.copy_blocks([l[0] for l in layers], [l[1] for l in layers], pairs)
    for (k0, v0), k1, v1 in zip(layers, ks, vs):
        assert np.array_equal(k1[3], k0[0]) and np.array_equal(k1[4], k0[3])   # reads before writes
        assert np.array_equal(v1[3], v0[0]) and np.array_equal(v1[4], v0[3])
        for b in (0, 1, 2):
            assert np.array_equal(k1[b], k0[b]) and np.array_equal(v1[b], v0[b])


def test_swap_blocks_matches_element_loop():
    rng = wl.rng_for(32)
    src = wl.bf16_normal(rng, (6, 2, 4, 3))          # e.g. the device pool
    dst = wl.bf16_normal(rng, (4, 2, 4, 3))          # e.g. a smaller host pool
    pairs = np.array([[5, 0], [1, 3], [5, 2]], np.int64)
    got = cache_ops.swap_blocks(src, dst, pairs)
    exp = dst.copy()
    for s_blk, d_blk in pairs:
        for h in range(2):
            for r in range(4):
                for d in range(3):
                    exp[d_blk, h, r, d] = src[s_blk, h, r, d]
    assert np.array_equal(got, exp) and np.array_equal(got[1], dst[1])


# ---------------------------------------------------------------------------
# Mutation tests: plausible mistakes planted in copies of the oracle source
# ---------------------------------------------------------------------------

MUTATIONS = {
    "drop_scale": ("z = float(scale) * (keys @ q)", "z = (keys @ q)"),
    "kv_head_modulo": ("kv_head = h // group", "kv_head = h % num_kv_heads"),
    "drop_current_token": ("length = int(context_lens[s])\n        if length == 0:",
                           "length = int(context_lens[s]) - 1\n        if length <= 0:"),
    "row_from_block_index": ("rows = positions % block_size", "rows = positions // block_size % block_size"),
    "table_by_row": ("physical = np.asarray(table_row)[positions // block_size]",
                     "physical = np.asarray(table_row)[positions % len(table_row)]"),
    "softmax_no_normalise": ("w = w / w.sum()", "w = w / len(w)"),
    "values_from_keys": ("out[s, h] = attend(q_all[s, h], keys[:, kv_head, :], values[:, kv_head, :], scale64)",
                         "out[s, h] = attend(q_all[s, h], keys[:, kv_head, :], keys[:, kv_head, :], scale64)"),
    "scale_squared": ("scale64 = float(np.float32(scale))\n    q_all",
                      "scale64 = float(np.float32(scale)) ** 2\n    q_all"),
}


def mutant(name):
    old, new = MUTATIONS[name]
    src = inspect.getsource(paged_attention)
    assert old in src, name
    ns = {}
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    return ns["paged_decode"]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name):
    impl = mutant(name)
    caught = []
    for pin in ATTENTION_PINS:
        try:
            ok = pin(impl)
        except Exception:
            ok = False
        if not ok:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutation {name}"


# ---------------------------------------------------------------------------
# The bf16 widening every attention oracle starts from
# ---------------------------------------------------------------------------

def pin_bf16_widening_every_pattern(widen):
    """All 65,536 bf16 bit patterns against torch's own bfloat16 -> float64 conversion
    (bf16 is the upper half of a float32, so widening is exact); NaN patterns must stay
    NaN, and the result keeps the input's shape."""
    bits = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    got = widen(bits.reshape(256, 256)).reshape(-1)
    nan = np.isnan(ref)
    return np.array_equal(nan, np.isnan(got)) and np.array_equal(ref[~nan], got[~nan])


def pin_bf16_widening_hand_cases(widen):
    """Worked by hand from the bf16 layout (1 sign, 8 exponent bits with bias 127, 7 mantissa bits)."""
    cases = {0x3F80: 1.0, 0xBF80: -1.0, 0x4000: 2.0, 0x3FC0: 1.5, 0x4049: 3.140625, 0x0001: 2.0 ** -133,
             0x7F7F: (2 - 2 ** -7) * 2.0 ** 127, 0x0000: 0.0, 0x7F80: math.inf, 0xFF80: -math.inf}
    got = widen(np.array(list(cases), dtype=np.uint16))
    return all(g == v for g, v in zip(got, cases.values()))


WIDEN_PINS = [pin_bf16_widening_every_pattern, pin_bf16_widening_hand_cases]


@pytest.mark.parametrize("pin", WIDEN_PINS, ids=lambda p: p.__name__)
def test_bf16_widening_pin(pin):
    assert pin(paged_attention.bf16_bits_to_f64)


WIDEN_MUTATIONS = {
    # the bits read as IEEE half precision instead of bfloat16
    "read_as_float16": ("return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)",
                        "return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)"),
    "shift_by_15": ("astype(np.uint32) << 16)", "astype(np.uint32) << 15)"),
}


@pytest.mark.parametrize("name", sorted(WIDEN_MUTATIONS))
def test_widening_pins_catch_planted_mistake(name):
    old, new = WIDEN_MUTATIONS[name]
    src = inspect.getsource(paged_attention)
    assert old in src, name
    ns = {}
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    caught = [p.__name__ for p in WIDEN_PINS if not _safe(p, ns["bf16_bits_to_f64"])]
    assert caught, f"no pin catches mutation {name}"


def _safe(pin, impl):
    try:
        return pin(impl)
    except Exception:
        return False
