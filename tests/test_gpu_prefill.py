"""paged_attention_prefill (tcgen05) on the GPU against the float64 prefill oracle.

Small batches cover every group size the kernel takes (g = 1 .. 128), both block
sizes, chunks that end inside a query tile, key tiles that cross the causal
diagonal, whole prompts and one-token chunks; full-size chunked-prefill batches
are checked on sampled rows.  Tolerance: max-abs 1e-2 and relative-L2 5e-3
against the oracle (fp32 output), as for decode."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import prefill as oracle
from tests.gpu_helpers import compare, dev_bf16

pytestmark = pytest.mark.gpu


class DevicePrefill:
    """A workloads.PrefillBatch resident on the GPU."""

    def __init__(self, b, key_cache=None, value_cache=None):
        self.b = b
        self.query = dev_bf16(b.query)
        self.key_cache = dev_bf16(b.key_cache) if key_cache is None else key_cache
        self.value_cache = dev_bf16(b.value_cache) if value_cache is None else value_cache
        self.tables = torch.from_numpy(np.ascontiguousarray(b.block_tables, np.int32)).cuda()
        self.qstart = torch.from_numpy(np.ascontiguousarray(b.query_start, np.int32)).cuda()
        self.lens = torch.from_numpy(np.ascontiguousarray(b.context_lens, np.int32)).cuda()

    def run(self, pkv, out_dtype=torch.float32, status=None, max_context_len=None, out=None, ws=None):
        b = self.b
        maxl = b.max_context_len if max_context_len is None else max_context_len
        if ws is None:
            ws = torch.empty(pkv.paged_attention_prefill_workspace_size(b.num_seqs, b.total_q, b.num_heads,
                                                                        b.num_kv_heads),
                             dtype=torch.uint8, device="cuda")
        if out is None:
            out = torch.empty((b.total_q, b.num_heads, b.head_dim), dtype=out_dtype, device="cuda")
        own = status is None
        if own:
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
        pkv.paged_attention_prefill(out, self.query, self.key_cache, self.value_cache, self.tables, self.qstart,
                                    self.lens, maxl, b.scale, ws, status=status)
        torch.cuda.synchronize()
        if own:
            assert status.item() == 0, f"device status {status.item():#x}"
        return out


def oracle_out(b):
    return oracle.paged_prefill(b.query, b.key_cache, b.value_cache, b.block_tables, b.query_start, b.context_lens,
                                b.scale)


CASES = {
    # name: make_prefill_batch arguments
    "mha_bs16": dict(name="chunked_prefill_13b", num_heads=4, num_kv_heads=4, query_lens=[1, 37, 128, 200],
                     earlier_lens=[0, 5, 300, 1000]),
    "mha_bs32": dict(name="chunked_prefill_13b", num_heads=2, num_kv_heads=2, block_size=32,
                     query_lens=[130, 64, 3], earlier_lens=[250, 0, 77]),
    "gqa2": dict(name="chunked_prefill_13b", num_heads=8, num_kv_heads=4, query_lens=[70, 129],
                 earlier_lens=[40, 400]),
    "gqa4": dict(name="chunked_prefill_13b", num_heads=8, num_kv_heads=2, query_lens=[33, 90, 1],
                 earlier_lens=[500, 31, 6]),
    "gqa8_bs32": dict(name="chunked_prefill_long_gqa", num_heads=16, num_kv_heads=2, query_lens=[50, 17],
                      earlier_lens=[700, 1200]),
    "gqa16": dict(name="chunked_prefill_long_gqa", num_heads=32, num_kv_heads=2, query_lens=[20, 9],
                  earlier_lens=[300, 640]),
    "gqa32": dict(name="chunked_prefill_13b", num_heads=32, num_kv_heads=1, query_lens=[11, 4], earlier_lens=[200, 0]),
    "gqa128": dict(name="chunked_prefill_13b", num_heads=128, num_kv_heads=1, query_lens=[3, 2], earlier_lens=[150, 1]),
    "whole_prompt": dict(name="chunked_prefill_13b", num_heads=2, num_kv_heads=1, query_lens=[700],
                         earlier_lens=[0]),
    "one_token_chunks": dict(name="chunked_prefill_13b", num_heads=4, num_kv_heads=2, query_lens=[1, 1, 1, 1],
                             earlier_lens=[0, 15, 128, 513]),
    "empty_chunks": dict(name="chunked_prefill_13b", num_heads=4, num_kv_heads=4, query_lens=[0, 45, 0, 12, 0],
                         earlier_lens=[10, 60, 0, 3, 99]),
    "drawn_small": dict(name="chunked_prefill_13b", num_seqs=5, num_heads=4, num_kv_heads=4, length_scale=0.06),
    "drawn_gqa_small": dict(name="chunked_prefill_long_gqa", num_seqs=3, num_heads=16, num_kv_heads=2,
                            length_scale=0.05),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_prefill_matches_oracle(pkv, case):
    b = wl.make_prefill_batch(**CASES[case])
    out = DevicePrefill(b).run(pkv)
    compare(out.cpu().numpy(), oracle_out(b))


def test_bf16_output_is_rounded_f32(pkv):
    b = wl.make_prefill_batch(**CASES["gqa4"])
    d = DevicePrefill(b)
    o32 = d.run(pkv, torch.float32)
    o16 = d.run(pkv, torch.bfloat16)
    assert torch.equal(o16, o32.to(torch.bfloat16))


def test_stale_nan_rows_do_not_leak(pkv):
    """Pool rows past every context end (and whole unused blocks) hold NaN: masked
    keys and zeroed value rows keep them out of every output."""
    b = wl.make_prefill_batch(**CASES["mha_bs16"])
    kc, vc = b.key_cache.copy(), b.value_cache.copy()
    used = set()
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        for t in range(L):
            used.add((int(b.block_tables[s][t // b.block_size]), t % b.block_size))
    nan = np.uint16(0x7FC0)
    for blk in range(b.num_blocks):
        for r in range(b.block_size):
            if (blk, r) not in used:
                kc[blk, :, r, :] = nan
                vc[blk, :, r, :] = nan
    b.key_cache, b.value_cache = kc, vc
    out = DevicePrefill(b).run(pkv)
    compare(out.cpu().numpy(), oracle_out(b))


def test_repeated_calls_reuse_workspace(pkv):
    b = wl.make_prefill_batch(**CASES["gqa2"])
    d = DevicePrefill(b)
    ws = torch.empty(pkv.paged_attention_prefill_workspace_size(b.num_seqs, b.total_q, b.num_heads, b.num_kv_heads),
                     dtype=torch.uint8, device="cuda")
    first = d.run(pkv, ws=ws)
    for _ in range(3):
        assert torch.equal(d.run(pkv, ws=ws), first)


def test_bad_context_and_block_are_flagged(pkv):
    b = wl.make_prefill_batch(**CASES["mha_bs16"])
    d = DevicePrefill(b)
    lens = b.context_lens.copy()
    lens[1] = b.query_lens[1] - 1                     # chunk longer than the context
    d.lens = torch.from_numpy(lens).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((b.total_q, b.num_heads, b.head_dim), 7.0, device="cuda")
    d.run(pkv, status=st, out=out)
    assert st.item() & pkv.PKV_DEV_BAD_CONTEXT
    rows = slice(int(b.query_start[1]), int(b.query_start[2]))
    assert torch.all(out[rows] == 0)
    ref = oracle_out(b)
    keep = np.r_[0:int(b.query_start[1]), int(b.query_start[2]):b.total_q]
    compare(out.cpu().numpy()[keep], ref[keep])
    # a table entry outside the pool
    d2 = DevicePrefill(b)
    tables = b.block_tables.copy()
    tables[3][2] = b.num_blocks + 5
    d2.tables = torch.from_numpy(tables).cuda()
    st.zero_()
    d2.run(pkv, status=st)
    assert st.item() & pkv.PKV_DEV_BAD_BLOCK


@pytest.mark.parametrize("name", sorted(wl.PREFILL_WORKLOADS))
def test_full_size_sampled_rows(pkv, name):
    """The full-size batch in the launch configuration the benchmark times; the
    oracle recomputes sampled rows (first, last and random rows of each sequence)."""
    b = wl.make_prefill_batch(name)
    out = DevicePrefill(b).run(pkv).cpu().numpy()
    rng = wl.rng_for(700)
    rows = []
    for s in range(b.num_seqs):
        q0, q1 = int(b.query_start[s]), int(b.query_start[s + 1])
        if q1 > q0:
            rows += [q0, q1 - 1, int(rng.integers(q0, q1))]
    rows = sorted(set(rows))
    ref = oracle.prefill_rows(b.query, b.key_cache, b.value_cache, b.block_tables, b.query_start, b.context_lens,
                              b.scale, rows)
    compare(out[rows], ref)


def test_zero_rows_is_a_no_op(pkv):
    b = wl.make_prefill_batch(**CASES["empty_chunks"])
    q = torch.empty((0, b.num_heads, b.head_dim), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((0, b.num_heads, b.head_dim), dtype=torch.float32, device="cuda")
    d = DevicePrefill(b)
    zeros = torch.zeros(b.num_seqs + 1, dtype=torch.int32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    pkv.paged_attention_prefill(out, q, d.key_cache, d.value_cache, d.tables, zeros, d.lens, b.max_context_len,
                                b.scale, ws)
    torch.cuda.synchronize()
