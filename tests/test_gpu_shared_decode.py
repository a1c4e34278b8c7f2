"""Shared-prefix decode (pkv_paged_attention_decode_shared) on the GPU against the
float64 oracle: the result must be that of plain decode attention over each row's
whole context (Outcome School explainer, "内存共享": the rows share blocks, not
results).  Batches: a shared system prompt (small and full size, sampled rows),
beam forks with copy-on-write after appends (nested segments), several key-chunk
sizes, block size 32, a batch with no sharing, and a plan that no longer fits the
lengths (flagged, zero output).  Tolerance: max-abs 1e-2, relative-L2 5e-3 (fp32
output), as for decode."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import paged_attention as oracle
from oracle.block_manager import BlockManagerModel
from tests.gpu_helpers import DeviceBatch, compare, dev_bf16

pytestmark = pytest.mark.gpu


def run_shared(pkv, db, key_chunk=0, out_dtype=torch.float32, lens=None, plan_lens=None, status=None):
    b = db.b
    plan_lens = b.context_lens if plan_lens is None else plan_lens
    plan, info = pkv.shared_plan(b.block_tables, plan_lens, b.num_heads, b.num_kv_heads, b.block_size,
                                 key_chunk=key_chunk)
    plan_d = torch.from_numpy(plan).cuda()
    ws = torch.empty(pkv.paged_attention_decode_shared_workspace_size(info, b.num_heads, b.num_kv_heads, b.head_dim),
                     dtype=torch.uint8, device="cuda")
    out = torch.full((b.num_seqs, b.num_heads, b.head_dim), float("nan"), dtype=out_dtype, device="cuda")
    own = status is None
    if own:
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_attention_decode_shared(out, db.query, db.key_cache, db.value_cache, db.tables,
                                      db.lens if lens is None else lens, b.scale, plan_d, info, ws, status=status)
    torch.cuda.synchronize()
    if own:
        assert status.item() == 0, f"device status {status.item():#x}"
    return out, info


def oracle_out(b, rows=None):
    rows = range(b.num_seqs) if rows is None else rows
    rows = list(rows)
    return oracle.paged_decode(b.query[rows], b.key_cache, b.value_cache, np.asarray(b.block_tables)[rows],
                               np.asarray(b.context_lens)[rows], b.scale)


class Batch:
    """A decode batch given by tables and lengths, with seeded N(0,1) bf16 data."""

    def __init__(self, tables, lens, nb, Hq, Hkv, bs, seed, D=128):
        rng = wl.rng_for(seed)
        self.num_seqs, self.num_heads, self.num_kv_heads, self.head_dim = len(lens), Hq, Hkv, D
        self.block_size, self.num_blocks = bs, nb
        self.block_tables = np.ascontiguousarray(tables, np.int32)
        self.context_lens = np.ascontiguousarray(lens, np.int32)
        self.max_context_len = int(self.context_lens.max())
        self.scale = wl.fp32_scale(D)
        self.query = wl.bf16_normal(rng, (self.num_seqs, Hq, D))
        self.key_cache = wl.bf16_normal(rng, (nb, Hkv, bs, D))
        self.value_cache = wl.bf16_normal(rng, (nb, Hkv, bs, D))


def beam_batch(seed, parents=5, beams=4, prompt_tokens=300, bs=16, steps=3, Hq=32, Hkv=8):
    """A prompt shared by every parent, each parent forked into adjacent beams, then
    appended tokens whose first step copies each shared partial last block."""
    rng = wl.rng_for(seed)
    nb = 1200
    m = BlockManagerModel(nb, bs, initial_order=rng.permutation(nb).astype(np.int32))
    lens = prompt_tokens + rng.integers(1, 400, size=parents)
    m.add_seq(0, int(lens[0]))
    prefix = m.tables[0][:prompt_tokens // bs]
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
    mb = max(len(m.tables[i]) for i in ids)
    t, l = m.export_tables(ids, mb)
    return Batch(t, l, nb, Hq, Hkv, bs, seed + 50)


@pytest.mark.parametrize("key_chunk", [0, 128, 256])
def test_shared_prompt_matches_oracle(pkv, key_chunk):
    b = wl.make_decode_batch("prefix_beams", num_seqs=12, length_scale=0.3)
    out, info = run_shared(pkv, DeviceBatch(b), key_chunk=key_chunk)
    assert info.num_segments == 1 and info.num_partials > 0
    compare(out.cpu().numpy(), oracle_out(b))


@pytest.mark.parametrize("steps", [0, 1, 3])
@pytest.mark.parametrize("heads", [(32, 8), (16, 8), (64, 4)])
def test_beam_forks_match_oracle(pkv, steps, heads):
    b = beam_batch(7 + steps, steps=steps, Hq=heads[0], Hkv=heads[1])
    out, info = run_shared(pkv, DeviceBatch(b))
    assert info.num_segments >= 1
    compare(out.cpu().numpy(), oracle_out(b))


def test_block_size_32(pkv):
    b = beam_batch(21, bs=32, prompt_tokens=320, steps=2)
    out, _ = run_shared(pkv, DeviceBatch(b))
    compare(out.cpu().numpy(), oracle_out(b))


def test_bf16_output_is_the_rounded_f32_output(pkv):
    b = beam_batch(5, steps=1)
    db = DeviceBatch(b)
    f32, _ = run_shared(pkv, db)
    bf16, _ = run_shared(pkv, db, out_dtype=torch.bfloat16)
    assert torch.equal(bf16, f32.to(torch.bfloat16))


def test_no_sharing_equals_decode(pkv):
    b = wl.make_decode_batch("long_trace", num_seqs=3, length_scale=0.06)
    db = DeviceBatch(b)
    out, info = run_shared(pkv, db)
    assert info.num_segments == 0
    compare(out.cpu().numpy(), oracle_out(b))


def test_full_size_shared_prompt_sampled(pkv):
    """The 128-sequence shared-prompt batch (1024-token prompt), sampled rows against the oracle."""
    b = wl.make_decode_batch("prefix_beams")
    out, info = run_shared(pkv, DeviceBatch(b))
    assert info.num_segments == 1 and info.shared_tokens == wl.PREFIX_TOKENS
    rows = sorted(wl.rng_for(3).choice(b.num_seqs, 6, replace=False).tolist())
    compare(out.cpu().numpy()[rows], oracle_out(b, rows))


def test_stale_plan_is_flagged_and_zeroed(pkv):
    """A plan made for other lengths: PKV_DEV_BAD_CONTEXT and zero rows, nothing read
    out of range."""
    b = beam_batch(9, steps=1)
    db = DeviceBatch(b)
    lens = b.context_lens.copy()
    lens[2] += 1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, _ = run_shared(pkv, db, lens=torch.from_numpy(lens).cuda(), status=status)
    assert status.item() & pkv.PKV_DEV_BAD_CONTEXT
    assert torch.all(out == 0)
    # the same workspace and plan work again with the right lengths
    out, _ = run_shared(pkv, db)
    compare(out.cpu().numpy(), oracle_out(b))


def test_runs_on_a_non_default_stream(pkv):
    b = beam_batch(11, steps=2)
    db = DeviceBatch(b)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out, _ = run_shared(pkv, db)
    compare(out.cpu().numpy(), oracle_out(b))


def test_two_calls_on_two_streams(pkv):
    """Two batches decoded on two caller streams without ordering between them: each call
    forks its shared phase onto the library's side stream and joins it back, so both
    results stay right."""
    b1, b2 = beam_batch(13, steps=1), beam_batch(14, steps=2)
    d1, d2 = DeviceBatch(b1), DeviceBatch(b2)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    outs = []
    for db, st in ((d1, s1), (d2, s2)):
        with torch.cuda.stream(st):
            b = db.b
            plan, info = pkv.shared_plan(b.block_tables, b.context_lens, b.num_heads, b.num_kv_heads, b.block_size)
            plan_d = torch.from_numpy(plan).cuda()
            ws = torch.empty(pkv.paged_attention_decode_shared_workspace_size(info, b.num_heads, b.num_kv_heads, 128),
                             dtype=torch.uint8, device="cuda")
            out = torch.empty((b.num_seqs, b.num_heads, 128), dtype=torch.float32, device="cuda")
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
            pkv.paged_attention_decode_shared(out, db.query, db.key_cache, db.value_cache, db.tables, db.lens, b.scale,
                                              plan_d, info, ws, status=status)
            outs.append((out, status, plan_d, ws))
    torch.cuda.synchronize()
    for (out, status, _, _), b in zip(outs, (b1, b2)):
        assert status.item() == 0
        compare(out.cpu().numpy(), oracle_out(b))


def test_long_remainders_match_oracle(pkv):
    """Private remainders past one 128-token tile go through the tensor-core decode (shorter ones
    through the CUDA-core decode, as in the beam batches here): a shared prompt with long remainders."""
    lens = 1024 + np.array([1100, 1350, 1600, 1200, 1500], np.int32)
    b = wl.make_decode_batch("prefix_beams", lengths=lens, seed=91)
    out, info = run_shared(pkv, DeviceBatch(b))
    assert info.num_segments == 1 and info.max_suffix_len > 1024
    compare(out.cpu().numpy(), oracle_out(b))
