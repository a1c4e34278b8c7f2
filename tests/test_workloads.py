"""The seeded input generators: determinism, shapes and the length mixes."""
import numpy as np

import workloads as wl


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 0.0], np.float32)
    bits = wl.f32_to_bf16_bits(x)
    back = (bits.astype(np.uint32) << 16).view(np.float32)
    assert back.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, 1.0, -2.5, 0.0]


def test_generators_are_deterministic():
    a = wl.make_decode_batch("llama7b", num_seqs=4, length_scale=0.05)
    b = wl.make_decode_batch("llama7b", num_seqs=4, length_scale=0.05)
    for f in ("context_lens", "block_tables", "query", "key_cache", "value_cache", "free_order"):
        assert np.array_equal(getattr(a, f), getattr(b, f))


def test_tiny_workload_shape():
    b = wl.make_decode_batch("tiny")
    assert b.context_lens.tolist() == [1, 7, 16, 33]
    assert (b.num_heads, b.num_kv_heads, b.head_dim, b.block_size, b.num_blocks) == (2, 2, 64, 16, 64)
    assert b.scale == 0.125
    assert sorted(b.free_order.tolist()) == list(range(64))
    used = np.concatenate([b.block_tables[s][:-(-L // 16)] for s, L in enumerate(b.context_lens)])
    assert len(set(used.tolist())) == 6


def test_mixed_lengths_statistics():
    lens = wl.draw_lengths("llama13b_mixed_bs16", wl.rng_for(5), 20000)
    long = lens >= 1000
    assert abs(long.mean() - 0.3) < 0.02
    assert abs(lens[~long].mean() - 50) < 3
    assert lens.min() >= 1 and lens.max() <= 2000


def test_full_size_tables_without_data():
    b = wl.make_decode_batch("llama13b_mixed_bs16", with_data=False)
    assert b.num_seqs == 256 and b.num_heads == 40
    need = -(-b.context_lens // 16)
    used = np.concatenate([b.block_tables[s][:n] for s, n in enumerate(need)])
    assert len(set(used.tolist())) == len(used) <= b.num_blocks
    assert b.num_blocks == int(np.ceil(1.2 * need.sum()))


def test_prefix_workload_shares_first_blocks():
    b = wl.make_decode_batch("prefix_beams", with_data=False)
    assert (b.context_lens >= 1034).all() and (b.context_lens <= 1524).all()
    assert (b.block_tables[:, :64] == b.block_tables[0, :64]).all()
    private = np.concatenate([b.block_tables[s][64:-(-L // 16)] for s, L in enumerate(b.context_lens)])
    assert len(set(private.tolist())) == len(private)
    assert not set(private.tolist()) & set(b.block_tables[0, :64].tolist())


def test_trace_events_are_seeded():
    p = wl.TraceParams(steps=10)
    assert wl.trace_events(p, 3) == wl.trace_events(p, 3)
    init, arr = wl.trace_events(p, 3)
    assert len(init) == 16 and all(5000 <= L <= 32000 for L, _ in init)
    assert len(arr) == 10
