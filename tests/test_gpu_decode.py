"""paged_attention_decode on the GPU against the float64 oracle.

Every workload is run at a size the oracle finishes in seconds (several tiles,
ragged tails, every split size), plus full-size workloads on sampled sequences.
Tolerance: max-abs 1e-2 and relative-L2 5e-3 against the oracle (fp32 output)."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import paged_attention as oracle
from tests.gpu_helpers import DeviceBatch, compare, dev_bf16, host_bits

pytestmark = pytest.mark.gpu

PATHS = {"simt": 1, "tensor": 2}


def path_applies(b, path):
    """The tensor-core path covers grouped heads (2 <= g <= 16) at head_dim 128."""
    g = b.num_heads // b.num_kv_heads
    if path == "tensor" and not (b.head_dim == 128 and 2 <= g <= 16):
        pytest.skip("tensor-core path needs grouped query heads and head_dim 128")


def oracle_out(b):
    return oracle.paged_decode(b.query, b.key_cache, b.value_cache, b.block_tables, b.context_lens, b.scale)


CASES = {
    "tiny": dict(name="tiny"),
    "llama7b": dict(name="llama7b", num_seqs=8, length_scale=0.25),
    "llama13b_bs16": dict(name="llama13b_mixed_bs16", num_seqs=24, length_scale=0.5),
    "llama13b_bs32": dict(name="llama13b_mixed_bs32", num_seqs=24, length_scale=0.5),
    "prefix_beams": dict(name="prefix_beams", num_seqs=12, length_scale=0.25),
    "long_trace": dict(name="long_trace", num_seqs=3, length_scale=0.08),
    "d64_bs32": dict(name="llama7b", num_seqs=6, length_scale=0.2, head_dim=64, block_size=32, num_heads=8,
                     num_kv_heads=8),
    "gqa2_bs16": dict(name="llama7b", num_seqs=6, length_scale=0.3, num_heads=8, num_kv_heads=4),
    "gqa16_bs32": dict(name="long_trace", num_seqs=2, length_scale=0.05, num_heads=32, num_kv_heads=2),
    "gqa8_d64": dict(name="llama7b", num_seqs=4, length_scale=0.2, head_dim=64, num_heads=16, num_kv_heads=2),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("path", sorted(PATHS))
def test_decode_matches_oracle(pkv, case, path):
    b = wl.make_decode_batch(**CASES[case])
    path_applies(b, path)
    out = DeviceBatch(b).decode(pkv, path=PATHS[path])
    compare(out.cpu().numpy(), oracle_out(b))


@pytest.mark.parametrize("partition", [64, 128, 256, 512, 1024, 2048])
@pytest.mark.parametrize("path", sorted(PATHS))
def test_split_sizes_agree(pkv, partition, path):
    """Split-context partitions of every size give the oracle's result (the CUDA-core
    path reads at most 32 table entries per item and refuses longer splits)."""
    heads = (4, 4) if path == "simt" else (16, 4)
    b = wl.make_decode_batch("llama7b", num_seqs=7, num_heads=heads[0], num_kv_heads=heads[1],
                             lengths=[1, 63, 64, 65, 129, 1500, 4500])
    if path == "simt" and partition // b.block_size > 32:
        with pytest.raises(pkv.PkvError) as e:
            DeviceBatch(b).decode(pkv, partition=partition, path=PATHS[path])
        assert e.value.code == pkv.PKV_ERR_UNSUPPORTED
        return
    ref = oracle_out(b)
    out = DeviceBatch(b).decode(pkv, partition=partition, path=PATHS[path])
    compare(out.cpu().numpy(), ref)


@pytest.mark.parametrize("path", sorted(PATHS))
def test_bf16_output_is_rounded_fp32(pkv, path):
    name = "llama13b_mixed_bs16" if path == "simt" else "prefix_beams"
    b = wl.make_decode_batch(name, num_seqs=16, length_scale=0.3)
    db = DeviceBatch(b)
    f32 = db.decode(pkv, out_dtype=torch.float32, path=PATHS[path])
    bf = db.decode(pkv, out_dtype=torch.bfloat16, path=PATHS[path])
    assert torch.equal(bf, f32.to(torch.bfloat16))


@pytest.mark.parametrize("path", sorted(PATHS))
def test_zero_length_and_single_token(pkv, path):
    b = wl.make_decode_batch("llama7b", num_seqs=4, num_heads=4, num_kv_heads=2, lengths=[0, 1, 0, 17])
    out = DeviceBatch(b).decode(pkv, path=PATHS[path]).cpu().numpy()
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    compare(out, oracle_out(b))
    # one token: the output is exactly that token's V (softmax weight 1)
    v = oracle.bf16_bits_to_f64(b.value_cache[b.block_tables[1][0], :, 0, :])
    assert np.array_equal(out[1], np.repeat(v, 2, axis=0))


@pytest.mark.parametrize("path", sorted(PATHS))
def test_runs_of_empty_contexts(pkv, path):
    """Runs of zero-length sequences between long ones (each gives one empty work item;
    the plan puts them last, right behind the longest items' final tiles)."""
    lengths = [0] * 6 + [700] + [0] * 9 + [1, 0, 0, 0, 0, 300, 0, 17] + [0] * 12 + [2049]
    b = wl.make_decode_batch("llama7b", num_heads=8, num_kv_heads=2 if path == "tensor" else 8, lengths=lengths)
    db = DeviceBatch(b)
    ref = oracle_out(b)
    for _ in range(3):
        out = db.decode(pkv, path=PATHS[path]).cpu().numpy()
        assert np.all(out[np.array(lengths) == 0] == 0)
        compare(out, ref)


@pytest.mark.parametrize("path", sorted(PATHS))
def test_stale_nan_rows_do_not_leak(pkv, path):
    """Rows past a context's end (stale pool rows) never enter the result, even as NaN."""
    b = wl.make_decode_batch("llama13b_mixed_bs32", num_seqs=8, num_heads=8, num_kv_heads=4 if path == "tensor" else 8,
                             length_scale=0.1)
    nan = np.uint16(0x7FC1)
    for s, L in enumerate(b.context_lens):
        last = b.block_tables[s][(L - 1) // b.block_size]
        b.key_cache[last, :, (L - 1) % b.block_size + 1:, :] = nan
        b.value_cache[last, :, (L - 1) % b.block_size + 1:, :] = nan
    out = DeviceBatch(b).decode(pkv, path=PATHS[path]).cpu().numpy()
    compare(out, oracle_out(b))


def test_permuted_pool_gives_same_output(pkv):
    """Blocks may sit anywhere in the pool: permuting physical blocks (and the tables
    with them) leaves the GPU output bit-identical."""
    b = wl.make_decode_batch("llama7b", num_seqs=6, num_heads=8, num_kv_heads=8, length_scale=0.2)
    base = DeviceBatch(b).decode(pkv)
    perm = wl.rng_for(5).permutation(b.num_blocks)
    kc, vc = np.empty_like(b.key_cache), np.empty_like(b.value_cache)
    kc[perm], vc[perm] = b.key_cache, b.value_cache
    b.key_cache, b.value_cache = kc, vc
    b.block_tables = perm[b.block_tables].astype(np.int32)
    assert torch.equal(base, DeviceBatch(b).decode(pkv))


@pytest.mark.parametrize("path", sorted(PATHS))
def test_bad_table_entry_and_context_are_flagged(pkv, path):
    heads = (2, 2) if path == "simt" else (8, 2)
    b = wl.make_decode_batch("llama7b", num_seqs=3, num_heads=heads[0], num_kv_heads=heads[1], lengths=[40, 20, 30])
    b.block_tables[0][1] = b.num_blocks + 5            # out of the pool
    db = DeviceBatch(b)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = db.decode(pkv, status=status, path=PATHS[path]).cpu().numpy()
    assert status.item() & pkv.PKV_DEV_BAD_BLOCK
    # sequences with valid tables are unaffected
    good = wl.make_decode_batch("llama7b", num_seqs=3, num_heads=heads[0], num_kv_heads=heads[1], lengths=[40, 20, 30])
    compare(out[1:], oracle_out(good)[1:])
    # a context longer than the bound: row zeroed, flagged
    db.lens[2] = 10_000
    status.zero_()
    out = db.decode(pkv, status=status, max_context_len=64, path=PATHS[path]).cpu().numpy()
    assert status.item() & pkv.PKV_DEV_BAD_CONTEXT
    assert np.all(out[2] == 0)


@pytest.mark.parametrize("path", sorted(PATHS))
def test_repeated_calls_reuse_workspace(pkv, path):
    """The arrival counters are re-armed by every call: back-to-back calls on one
    workspace give identical outputs."""
    b = wl.make_decode_batch("long_trace", num_seqs=2, length_scale=0.05)
    db = DeviceBatch(b)
    maxl = b.max_context_len
    ws = torch.empty(pkv.paged_attention_workspace_size(2, 64, 8, 128, 32, maxl, 64), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        out = torch.empty((2, 64, 128), dtype=torch.float32, device="cuda")
        pkv.paged_attention_decode(out, db.query, db.key_cache, db.value_cache, db.tables, db.lens, maxl, b.scale, ws,
                                   partition_tokens=64, path=PATHS[path])
        outs.append(out)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    compare(outs[0].cpu().numpy(), oracle_out(b))


@pytest.mark.parametrize("path", sorted(PATHS))
def test_longest_context(pkv, path):
    """One 131072-token context (4096 blocks of 32): 256 partitions of 512 tokens on the
    CUDA-core path, 64 of 2048 on the tensor path, merged into one row per head."""
    L = 131072
    heads = (4, 4) if path == "simt" else (32, 4)
    b = wl.make_decode_batch("long_trace", num_seqs=1, num_heads=heads[0], num_kv_heads=heads[1], lengths=[L],
                             pool_factor=1.0, with_data=False)
    rng = wl.rng_for(310)
    b.query = wl.bf16_normal(rng, (1, b.num_heads, 128))
    shape = (b.num_blocks, b.num_kv_heads, b.block_size, 128)
    kc, vc = device_pool(shape, 3), device_pool(shape, 4)
    part = 512 if path == "simt" else 2048
    out = DeviceBatch(b, kc, vc).decode(pkv, partition=part, path=PATHS[path]).cpu().numpy()
    compare(out, sampled_oracle(b, kc, vc, [0]))


# ---------------------------------------------------------------------------
# Full-size workloads: sampled sequences checked one by one against the oracle
# ---------------------------------------------------------------------------

def device_pool(shape, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)


def sampled_oracle(b, kc_dev, vc_dev, seqs):
    """Oracle on the listed sequences, with their blocks copied out of the device pool
    (pool contents come from torch's seeded generator, untouched by the library)."""
    rows = []
    for s in seqs:
        need = -(-int(b.context_lens[s]) // b.block_size)
        blocks = b.block_tables[s][:need]
        kc = host_bits(kc_dev[torch.from_numpy(blocks.astype(np.int64)).cuda()])
        vc = host_bits(vc_dev[torch.from_numpy(blocks.astype(np.int64)).cuda()])
        table = np.arange(need, dtype=np.int32)[None, :]
        rows.append(oracle.paged_decode(b.query[s:s + 1], kc, vc, table, b.context_lens[s:s + 1], b.scale)[0])
    return np.stack(rows)


@pytest.mark.parametrize("name", ["llama7b", "llama13b_mixed_bs16", "llama13b_mixed_bs32", "prefix_beams",
                                  "long_trace"])
@pytest.mark.parametrize("path", sorted(PATHS))
def test_full_size_sampled(pkv, name, path):
    b = wl.make_decode_batch(name, with_data=False)
    path_applies(b, path)
    rng = wl.rng_for(300)
    b.query = wl.bf16_normal(rng, (b.num_seqs, b.num_heads, b.head_dim))
    shape = (b.num_blocks, b.num_kv_heads, b.block_size, b.head_dim)
    kc, vc = device_pool(shape, 1), device_pool(shape, 2)
    out = DeviceBatch(b, kc, vc).decode(pkv, path=PATHS[path]).cpu().numpy()
    assert np.all(np.isfinite(out))
    order = np.argsort(b.context_lens)
    seqs = sorted(set([int(order[0]), int(order[-1]), int(order[len(order) // 2])] +
                      rng.choice(b.num_seqs, size=min(5, b.num_seqs), replace=False).tolist()))
    compare(out[seqs], sampled_oracle(b, kc, vc, seqs))
