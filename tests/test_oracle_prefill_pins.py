"""Pins for the prefill / chunked-prefill attention oracle (CPU only).

The oracle is tied to: torch's causal scaled_dot_product_attention in float64
(a whole prompt in one call), the decode oracle (a one-token chunk), chunking
invariance (a prompt prefilled in pieces gives the rows of the one-call prefill),
and a closed form (equal keys: row p averages values 0..p).  Mutation tests plant
plausible mistakes in copies of the oracle's source.
"""
import inspect

import numpy as np
import pytest
import torch

import workloads as wl
from oracle import paged_attention, prefill

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def pool_from_contiguous(k_bits, v_bits, lens, bs, seed):
    """Scatter contiguous per-sequence K/V [B, Hkv, Lmax, D] into a shuffled pool."""
    B, Hkv, _, D = k_bits.shape
    need = -(-np.asarray(lens) // bs)
    nb = int(need.sum()) + 3
    rng = wl.rng_for(seed)
    order = rng.permutation(nb).astype(np.int32)
    tables = wl.place_blocks(np.asarray(lens, np.int32), bs, order)
    kc = wl.bf16_normal(rng, (nb, Hkv, bs, D))
    vc = wl.bf16_normal(rng, (nb, Hkv, bs, D))
    for s in range(B):
        for t in range(int(lens[s])):
            kc[tables[s][t // bs], :, t % bs] = k_bits[s, :, t]
            vc[tables[s][t // bs], :, t % bs] = v_bits[s, :, t]
    return kc, vc, tables


def case(seed, lens, qlens, Hq=4, Hkv=2, D=16, bs=4):
    rng = wl.rng_for(seed)
    lens = np.asarray(lens, np.int32)
    qlens = np.asarray(qlens, np.int32)
    L = int(lens.max())
    k = wl.bf16_normal(rng, (len(lens), Hkv, L, D))
    v = wl.bf16_normal(rng, (len(lens), Hkv, L, D))
    kc, vc, tables = pool_from_contiguous(k, v, lens, bs, seed + 1)
    qstart = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = wl.bf16_normal(rng, (int(qstart[-1]), Hq, D))
    return dict(q=q, k=k, v=v, kc=kc, vc=vc, tables=tables, lens=lens, qlens=qlens, qstart=qstart,
                scale=wl.fp32_scale(D), bs=bs)


def run(impl, c, **over):
    d = dict(c, **over)
    return impl(d["q"], d["kc"], d["vc"], d["tables"], d["qstart"], d["lens"], d["scale"])


# ---------------------------------------------------------------------------

def pin_library_causal(impl):
    """Whole prompts (chunk = context): torch's is_causal attention in float64."""
    c = case(1, lens=[5, 11, 8], qlens=[5, 11, 8], Hq=6, Hkv=2)
    got = run(impl, c)
    g = 3
    for s in range(3):
        L = int(c["lens"][s])
        q = torch.from_numpy(f64(c["q"][c["qstart"][s]:c["qstart"][s + 1]])).transpose(0, 1)  # [Hq, L, D]
        k = torch.from_numpy(f64(c["k"][s, :, :L])).repeat_interleave(g, 0)
        v = torch.from_numpy(f64(c["v"][s, :, :L])).repeat_interleave(g, 0)
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True,
                                                               scale=float(np.float32(c["scale"])))
        if not np.allclose(got[c["qstart"][s]:c["qstart"][s + 1]], ref.transpose(0, 1).numpy(), rtol=0, atol=1e-12):
            return False
    return True


def pin_one_token_is_decode(impl):
    """A one-token chunk is a decode step over the whole context."""
    c = case(2, lens=[1, 9, 14, 6], qlens=[1, 1, 1, 1])
    got = run(impl, c)
    ref = paged_attention.paged_decode(c["q"], c["kc"], c["vc"], c["tables"], c["lens"], c["scale"])
    return np.allclose(got, ref, rtol=0, atol=1e-13)


def pin_chunking_invariance(impl):
    """Prefilling a 23-token prompt as chunks 7 + 9 + 7 gives the rows of one call."""
    c = case(3, lens=[23], qlens=[23])
    whole = run(impl, c)
    rows = []
    for lo, hi in ((0, 7), (7, 16), (16, 23)):
        part = dict(c)
        part["q"] = c["q"][lo:hi]
        part["lens"] = np.array([hi], np.int32)
        part["qstart"] = np.array([0, hi - lo], np.int32)
        rows.append(run(impl, part))
    return np.allclose(np.concatenate(rows), whole, rtol=0, atol=1e-13)


def pin_equal_keys_running_mean(impl):
    """All keys of a sequence equal: chunk row at position p is the mean of values 0..p."""
    c = case(4, lens=[13, 10], qlens=[6, 10])
    k = c["k"].copy()
    k[:] = c["k"][:, :, :1, :]
    kc, vc, tables = pool_from_contiguous(k, c["v"], c["lens"], c["bs"], 40)
    got = run(impl, c, kc=kc, vc=vc, tables=tables)
    for s in range(2):
        n, L = int(c["qlens"][s]), int(c["lens"][s])
        for i in range(n):
            p = L - n + i
            for h in range(4):
                expect = f64(c["v"][s, h // 2, :p + 1]).mean(axis=0)
                if not np.allclose(got[c["qstart"][s] + i, h], expect, rtol=0, atol=1e-13):
                    return False
    return True


def pin_empty_chunks(impl):
    """Sequences with no new tokens own no rows; the others are unaffected."""
    c = case(5, lens=[7, 9, 12], qlens=[3, 0, 4])
    got = run(impl, c)
    solo = case(5, lens=[7, 9, 12], qlens=[3, 0, 4])
    a = run(impl, dict(solo, q=solo["q"][:3], lens=solo["lens"][:1], qstart=np.array([0, 3], np.int32),
                       tables=solo["tables"][:1]))
    return got.shape[0] == 7 and np.allclose(got[:3], a, rtol=0, atol=1e-13)


PREFILL_PINS = [pin_library_causal, pin_one_token_is_decode, pin_chunking_invariance, pin_equal_keys_running_mean,
                pin_empty_chunks]


@pytest.mark.parametrize("pin", PREFILL_PINS, ids=lambda p: p.__name__)
def test_prefill_oracle_pin(pin):
    assert pin(prefill.paged_prefill)


def test_prefill_rows_matches_whole_call():
    c = case(6, lens=[9, 20, 4, 15], qlens=[9, 5, 0, 7], Hq=4, Hkv=1)
    whole = run(prefill.paged_prefill, c)
    rows = [0, 4, 8, 9, 13, 14, 17, 20]
    got = prefill.prefill_rows(c["q"], c["kc"], c["vc"], c["tables"], c["qstart"], c["lens"], c["scale"], rows)
    assert np.allclose(got, whole[rows], rtol=0, atol=1e-13)


MUTATIONS = {
    "exclude_self": ("keys[:position + 1, kv_head, :]", "keys[:position, kv_head, :]"),
    "position_from_chunk_start": ("position = length - n + i", "position = i"),
    "kv_head_modulo": ("kv_head = h // group", "kv_head = h % num_kv_heads"),
    "row_ignores_packing": ("row = starts[s] + i", "row = i"),
    "values_window_whole_context": ("values[:position + 1, kv_head, :]", "values[:, kv_head, :][:position + 1][::-1]"),
}


def mutant(name):
    old, new = MUTATIONS[name]
    src = inspect.getsource(prefill)
    assert old in src, name
    src = src.replace("from .paged_attention import", "from oracle.paged_attention import")
    ns = {}
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    return ns["paged_prefill"]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_prefill_pins_catch_planted_mistake(name):
    impl = mutant(name)
    caught = []
    for pin in PREFILL_PINS:
        try:
            ok = pin(impl)
        except Exception:
            ok = False
        if not ok:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutation {name}"
