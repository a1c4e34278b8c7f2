"""The 8-bit (e4m3) KV cache on the GPU against the oracle.

reshape_and_cache_fp8 is checked bit for bit on every bf16 bit pattern and on
drawn K/V; paged_attention_decode_fp8 on seeded e4m3 pools (drawn as bit
patterns) with per-kv-head scales, at oracle-sized batches and on sampled
sequences of the full-size 13B batch.  Attention tolerance as for bf16 decode."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import fp8 as oracle
from tests.gpu_helpers import compare, dev_bf16

pytestmark = pytest.mark.gpu


def u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.uint8)).cuda()


def f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def same_codes(got, ref):
    """Equal codes; a NaN result may carry either sign."""
    nan_g = (got & 0x7F) == 0x7F
    nan_r = (ref & 0x7F) == 0x7F
    return np.array_equal(nan_g, nan_r) and np.array_equal(got[~nan_g], ref[~nan_r])


@pytest.mark.parametrize("scale", [1.0, 0.0173, 2.0 ** -6, 3.3])
def test_cache_write_every_bf16_value(pkv, scale):
    """All 65536 bf16 bit patterns (zeros, subnormals, the saturating range, inf, NaN)."""
    Hkv, D, bs = 2, 128, 16
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    T = 65536 // (Hkv * D)
    k = bits.reshape(T, Hkv, D)
    v = bits[::-1].copy().reshape(T, Hkv, D)
    nb = T // bs
    slots = np.arange(T, dtype=np.int64)[::-1].copy()
    ks = np.array([scale, scale * 0.5], np.float32)
    vs = np.array([scale * 2, scale], np.float32)
    kc, vc = u8(np.zeros((nb, Hkv, bs, D))), u8(np.zeros((nb, Hkv, bs, D)))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.reshape_and_cache_fp8(dev_bf16(k), dev_bf16(v), kc, vc, torch.from_numpy(slots).cuda(), f32(ks), f32(vs),
                              status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ek, ev = oracle.reshape_and_cache_fp8(k, v, np.zeros((nb, Hkv, bs, D), np.uint8),
                                          np.zeros((nb, Hkv, bs, D), np.uint8), slots, ks, vs)
    assert same_codes(kc.cpu().numpy(), ek) and same_codes(vc.cpu().numpy(), ev)


def test_cache_write_skips_and_flags(pkv):
    rng = wl.rng_for(810)
    T, Hkv, D, bs, nb = 9, 4, 128, 32, 3
    k, v = wl.new_tokens(rng, T, Hkv, D)
    start = wl.e4m3_codes(rng, (nb, Hkv, bs, D))
    kc, vc = u8(start), u8(start)
    slots = np.array([0, -1, 95, 3, nb * bs, 40, -5, 64, 31], np.int64)
    ks = wl.kv_scales(rng, Hkv)
    vs = wl.kv_scales(rng, Hkv)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.reshape_and_cache_fp8(dev_bf16(k), dev_bf16(v), kc, vc, torch.from_numpy(slots).cuda(), f32(ks), f32(vs),
                              status=st)
    torch.cuda.synchronize()
    assert st.item() & pkv.PKV_DEV_BAD_SLOT
    keep = np.where(slots < nb * bs, slots, -1)
    ek, ev = oracle.reshape_and_cache_fp8(k, v, start, start, keep, ks, vs)
    assert np.array_equal(kc.cpu().numpy(), ek) and np.array_equal(vc.cpu().numpy(), ev)


def fp8_batch(name, seed=820, **kw):
    """A decode batch whose pool is drawn as e4m3 codes, with per-kv-head scales."""
    b = wl.make_decode_batch(name, with_data=False, **kw)
    rng = wl.rng_for(seed)
    b.query = wl.bf16_normal(rng, (b.num_seqs, b.num_heads, b.head_dim))
    kc = wl.e4m3_codes(rng, (b.num_blocks, b.num_kv_heads, b.block_size, b.head_dim))
    vc = wl.e4m3_codes(rng, (b.num_blocks, b.num_kv_heads, b.block_size, b.head_dim))
    return b, kc, vc, wl.kv_scales(rng, b.num_kv_heads), wl.kv_scales(rng, b.num_kv_heads)


PATHS = {"simt": 1, "tensor": 2}


def path_applies(b, path):
    """The 8-bit tensor-core path covers grouped heads (2 <= g <= 16); head_dim is 128."""
    g = b.num_heads // b.num_kv_heads
    if path == "tensor" and not 2 <= g <= 16:
        pytest.skip("tensor-core path needs grouped query heads")


def run_fp8(pkv, b, kc, vc, ks, vs, out_dtype=torch.float32, partition=0, path=0, status_ok=True, max_len=None):
    maxl = b.max_context_len if max_len is None else max_len
    ws = torch.empty(pkv.paged_attention_workspace_size(b.num_seqs, b.num_heads, b.num_kv_heads, b.head_dim,
                                                        b.block_size, maxl, partition),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty((b.num_seqs, b.num_heads, b.head_dim), dtype=out_dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kc_d = kc if isinstance(kc, torch.Tensor) else u8(kc)
    vc_d = vc if isinstance(vc, torch.Tensor) else u8(vc)
    pkv.paged_attention_decode_fp8(out, dev_bf16(b.query), kc_d, vc_d, f32(ks), f32(vs),
                                   torch.from_numpy(np.ascontiguousarray(b.block_tables)).cuda(),
                                   torch.from_numpy(np.ascontiguousarray(b.context_lens)).cuda(), maxl, b.scale, ws,
                                   partition_tokens=partition, path=path, status=st)
    torch.cuda.synchronize()
    if status_ok:
        assert st.item() == 0
        return out
    return out, st.item()


def oracle_fp8(b, kc, vc, ks, vs):
    return oracle.paged_decode_fp8(b.query, kc, vc, ks, vs, b.block_tables, b.context_lens, b.scale)


CASES = {
    "llama7b": dict(name="llama7b", num_seqs=8, length_scale=0.25),
    "llama13b_bs16": dict(name="llama13b_mixed_bs16", num_seqs=24, length_scale=0.5),
    "llama13b_bs32": dict(name="llama13b_mixed_bs32", num_seqs=24, length_scale=0.5),
    "gqa_prefix": dict(name="prefix_beams", num_seqs=12, length_scale=0.25),
    "gqa_long": dict(name="long_trace", num_seqs=3, length_scale=0.08),
    "gqa2_bs16": dict(name="llama7b", num_seqs=6, length_scale=0.3, num_heads=8, num_kv_heads=4),
    "gqa4_bs32": dict(name="llama13b_mixed_bs32", num_seqs=10, length_scale=0.3, num_heads=16, num_kv_heads=4),
    "gqa16_bs32": dict(name="long_trace", num_seqs=2, length_scale=0.05, num_heads=32, num_kv_heads=2),
    "gqa5": dict(name="llama7b", num_seqs=5, length_scale=0.3, num_heads=10, num_kv_heads=2),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("path", sorted(PATHS))
def test_decode_fp8_matches_oracle(pkv, case, path):
    b, kc, vc, ks, vs = fp8_batch(**CASES[case])
    path_applies(b, path)
    out = run_fp8(pkv, b, kc, vc, ks, vs, path=PATHS[path])
    compare(out.cpu().numpy(), oracle_fp8(b, kc, vc, ks, vs))


def test_decode_fp8_paths_agree_on_auto(pkv):
    """PATH_AUTO takes the tensor cores for grouped heads: bit-identical to PATH_TENSOR."""
    b, kc, vc, ks, vs = fp8_batch(**CASES["gqa_prefix"])
    assert torch.equal(run_fp8(pkv, b, kc, vc, ks, vs), run_fp8(pkv, b, kc, vc, ks, vs, path=PATHS["tensor"]))


@pytest.mark.parametrize("partition", [64, 256, 512, 1024, 2048])
@pytest.mark.parametrize("path", sorted(PATHS))
def test_decode_fp8_split_sizes(pkv, partition, path):
    b, kc, vc, ks, vs = fp8_batch("llama7b", num_seqs=7, num_heads=8, num_kv_heads=2,
                                  lengths=[1, 63, 64, 65, 129, 1500, 4500])
    if path == "simt" and partition // b.block_size > 32:
        with pytest.raises(pkv.PkvError) as e:
            run_fp8(pkv, b, kc, vc, ks, vs, partition=partition, path=PATHS[path])
        assert e.value.code == pkv.PKV_ERR_UNSUPPORTED
        return
    out = run_fp8(pkv, b, kc, vc, ks, vs, partition=partition, path=PATHS[path])
    compare(out.cpu().numpy(), oracle_fp8(b, kc, vc, ks, vs))


@pytest.mark.parametrize("path", sorted(PATHS))
def test_decode_fp8_large_query_values(pkv, path):
    """Query components of 2^15 and more (beyond f16) take the scaled-query route; a
    kv head whose queries are all small keeps the unscaled route."""
    b, kc, vc, ks, vs = fp8_batch("llama7b", num_seqs=4, num_heads=8, num_kv_heads=4, length_scale=0.1)
    q = b.query.copy()
    q[1, 2, 5] = wl.f32_to_bf16_bits(np.array([70000.0], np.float32))[0]
    q[1, 7, 9] = wl.f32_to_bf16_bits(np.array([-40000.0], np.float32))[0]
    q[2, 0, :] = wl.f32_to_bf16_bits(np.full(128, 1.0e-3, np.float32))
    b.query = q
    ks = np.full_like(ks, 1e-6)                     # keep the scores in a sane range
    out = run_fp8(pkv, b, kc, vc, ks, vs, path=PATHS[path])
    compare(out.cpu().numpy(), oracle_fp8(b, kc, vc, ks, vs))


@pytest.mark.parametrize("path", sorted(PATHS))
def test_decode_fp8_bf16_output_is_rounded_f32(pkv, path):
    b, kc, vc, ks, vs = fp8_batch("llama7b", num_seqs=6, num_heads=8, num_kv_heads=8 if path == "simt" else 2,
                                  length_scale=0.2)
    o32 = run_fp8(pkv, b, kc, vc, ks, vs, torch.float32, path=PATHS[path])
    o16 = run_fp8(pkv, b, kc, vc, ks, vs, torch.bfloat16, path=PATHS[path])
    assert torch.equal(o16, o32.to(torch.bfloat16))


@pytest.mark.parametrize("path", sorted(PATHS))
def test_decode_fp8_runs_of_empty_contexts(pkv, path):
    """Runs of zero-length sequences between long ones (each gives one empty work item;
    the plan puts them last, right behind the longest items' final tiles)."""
    lengths = [0] * 6 + [700] + [0] * 9 + [1, 0, 0, 0, 0, 300, 0, 17] + [0] * 12 + [2049]
    b, kc, vc, ks, vs = fp8_batch("llama7b", num_heads=8, num_kv_heads=2, lengths=lengths)
    for _ in range(3):
        out = run_fp8(pkv, b, kc, vc, ks, vs, path=PATHS[path]).cpu().numpy()
        assert np.all(out[np.array(lengths) == 0] == 0)
        compare(out, oracle_fp8(b, kc, vc, ks, vs))


@pytest.mark.parametrize("path", sorted(PATHS))
def test_decode_fp8_one_token_is_its_value(pkv, path):
    b, kc, vc, ks, vs = fp8_batch("llama7b", num_heads=8, num_kv_heads=2, lengths=[1, 5, 1])
    out = run_fp8(pkv, b, kc, vc, ks, vs, path=PATHS[path]).cpu().numpy()
    v = oracle.e4m3_to_f64(vc[b.block_tables[0][0], :, 0, :]) * vs.astype(np.float64)[:, None]
    assert np.allclose(out[0], np.repeat(v, 4, axis=0), rtol=0, atol=1e-6 * np.abs(v).max())


@pytest.mark.parametrize("path", sorted(PATHS))
def test_decode_fp8_stale_nan_codes_do_not_leak(pkv, path):
    """Pool rows past a context's end may hold the NaN code; they never enter the result."""
    b, kc, vc, ks, vs = fp8_batch("llama13b_mixed_bs32", num_seqs=8, num_heads=8, num_kv_heads=2, length_scale=0.1)
    for s, L in enumerate(b.context_lens):
        last = b.block_tables[s][(L - 1) // b.block_size]
        kc[last, :, (L - 1) % b.block_size + 1:, :] = 0x7F
        vc[last, :, (L - 1) % b.block_size + 1:, :] = 0xFF
    out = run_fp8(pkv, b, kc, vc, ks, vs, path=PATHS[path])
    compare(out.cpu().numpy(), oracle_fp8(b, kc, vc, ks, vs))


@pytest.mark.parametrize("path", sorted(PATHS))
def test_decode_fp8_bad_table_entry_and_context_are_flagged(pkv, path):
    b, kc, vc, ks, vs = fp8_batch("llama7b", num_heads=8, num_kv_heads=2, lengths=[40, 20, 30])
    good = b.block_tables.copy()
    b.block_tables[0][1] = b.num_blocks + 5
    out, st = run_fp8(pkv, b, kc, vc, ks, vs, path=PATHS[path], status_ok=False)
    assert st & pkv.PKV_DEV_BAD_BLOCK
    b.block_tables = good
    compare(out.cpu().numpy()[1:], oracle_fp8(b, kc, vc, ks, vs)[1:])
    b.context_lens = np.array([40, 20, 10_000], np.int32)
    out, st = run_fp8(pkv, b, kc, vc, ks, vs, path=PATHS[path], status_ok=False, max_len=64)
    assert st & pkv.PKV_DEV_BAD_CONTEXT
    assert np.all(out.cpu().numpy()[2] == 0)


def device_codes(shape, seed):
    """e4m3 codes drawn on the device by torch's seeded generator (never NaN;
    magnitudes 2^-2 .. 2^3 before the scale)."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    sign = torch.randint(0, 2, shape, generator=g, device="cuda", dtype=torch.uint8)
    exp = torch.randint(5, 11, shape, generator=g, device="cuda", dtype=torch.uint8)
    mant = torch.randint(0, 8, shape, generator=g, device="cuda", dtype=torch.uint8)
    return (sign << 7) | (exp << 3) | mant


@pytest.mark.parametrize("name", ["llama13b_mixed_bs16", "prefix_beams", "long_trace"])
@pytest.mark.parametrize("path", sorted(PATHS))
def test_decode_fp8_full_size_sampled(pkv, name, path):
    b = wl.make_decode_batch(name, with_data=False)
    path_applies(b, path)
    rng = wl.rng_for(830)
    b.query = wl.bf16_normal(rng, (b.num_seqs, b.num_heads, b.head_dim))
    ks, vs = wl.kv_scales(rng, b.num_kv_heads), wl.kv_scales(rng, b.num_kv_heads)
    shape = (b.num_blocks, b.num_kv_heads, b.block_size, b.head_dim)
    kc, vc = device_codes(shape, 11), device_codes(shape, 12)
    out = run_fp8(pkv, b, kc, vc, ks, vs, path=PATHS[path]).cpu().numpy()
    assert np.all(np.isfinite(out))
    order = np.argsort(b.context_lens)
    seqs = sorted(set([int(order[0]), int(order[-1])] + [int(s) for s in rng.choice(b.num_seqs, 6, replace=False)]))
    rows = []
    for s in seqs:
        # the oracle on this sequence's blocks, copied out of the device pool
        need = -(-int(b.context_lens[s]) // b.block_size)
        blocks = torch.from_numpy(b.block_tables[s][:need].astype(np.int64)).cuda()
        table = np.arange(need, dtype=np.int32)[None, :]
        rows.append(oracle.paged_decode_fp8(b.query[s:s + 1], kc[blocks].cpu().numpy(), vc[blocks].cpu().numpy(),
                                            ks, vs, table, b.context_lens[s:s + 1], b.scale)[0])
    compare(out[seqs], np.stack(rows))


# ---- swap_blocks ---------------------------------------------------------------------

def test_swap_blocks_device_host_round_trip(pkv):
    from oracle import cache_ops
    rng = wl.rng_for(840)
    NB, HB, Hkv, bs, D = 20, 12, 2, 16, 128
    dev = wl.bf16_normal(rng, (NB, Hkv, bs, D))
    host0 = wl.bf16_normal(rng, (HB, Hkv, bs, D))
    d = dev_bf16(dev)
    h = torch.from_numpy(host0.view(np.int16)).view(torch.bfloat16).pin_memory()
    out_pairs = np.array([[3, 0], [17, 5], [0, 11], [9, 2]], np.int64)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.swap_blocks(d, h, torch.from_numpy(out_pairs).cuda(), status=st)
    torch.cuda.synchronize()
    host1 = cache_ops.swap_blocks(dev, host0, out_pairs)
    assert np.array_equal(h.view(torch.int16).numpy().view(np.uint16), host1)
    # back in, to other device blocks, with the pairs themselves in pinned host memory
    in_pairs = torch.from_numpy(np.array([[0, 1], [5, 19], [11, 7]], np.int64)).pin_memory()
    pkv.swap_blocks(h, d, in_pairs, status=st)
    torch.cuda.synchronize()
    dev1 = cache_ops.swap_blocks(host1, dev, in_pairs.numpy())
    assert st.item() == 0
    assert np.array_equal(d.view(torch.int16).cpu().numpy().view(np.uint16), dev1)
    # an 8-bit pool moves the same way
    codes = wl.e4m3_codes(rng, (NB, Hkv, bs, D))
    d8 = u8(codes)
    h8 = torch.zeros((HB, Hkv, bs, D), dtype=torch.uint8).pin_memory()
    pkv.swap_blocks(d8, h8, torch.from_numpy(out_pairs).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(h8.numpy(), cache_ops.swap_blocks(codes, np.zeros_like(h8.numpy()), out_pairs))


def test_swap_blocks_rejects_pageable_memory_and_flags_bad_pairs(pkv):
    d = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    pageable = torch.zeros((4, 256), dtype=torch.bfloat16)
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    with pytest.raises(pkv.PkvError) as e:
        pkv.library()  # the binding refuses non-pinned host tensors itself; go through the C ABI
        import ctypes
        rc = pkv.library().pkv_swap_blocks(ctypes.c_void_p(d.data_ptr()), ctypes.c_void_p(pageable.data_ptr()),
                                           ctypes.c_void_p(pairs.data_ptr()), 1, 4, 4, 512, None, None)
        pkv._check(rc, "swap_blocks")
    assert e.value.code == pkv.PKV_ERR_INVALID
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    h = torch.zeros((4, 256), dtype=torch.bfloat16).pin_memory()
    pkv.swap_blocks(d, h, torch.tensor([[0, 1], [7, 2], [1, -1]], dtype=torch.int64, device="cuda"), status=st)
    torch.cuda.synchronize()
    assert st.item() & pkv.PKV_DEV_BAD_PAIR
