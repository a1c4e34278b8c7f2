"""Calls on two caller streams at once.

Each call chains its kernels (plan, decode, merge; plan, query split, 8-bit decode, merge;
prefill plan, prefill), each later kernel launched to start while the one before it ends.
Two batches are decoded repeatedly on two streams with no ordering between them, each with
its own workspace; every output must be byte-for-byte the output of the same call run alone:
items are claimed dynamically, but each item's arithmetic, and the merge's partition order,
do not depend on which CTA runs it or on what runs beside it."""
import numpy as np
import pytest
import torch

import workloads as wl
from tests.gpu_helpers import DeviceBatch, dev_bf16
from tests.test_gpu_fp8 import f32, fp8_batch, u8

pytestmark = pytest.mark.gpu

PATH_SIMT, PATH_TENSOR = 1, 2
REPS = 6


def _run_two_streams(make_call, out_a, out_b):
    """make_call(which, out) returns a callable that enqueues one call on the current stream."""
    ref_a, ref_b = torch.empty_like(out_a), torch.empty_like(out_b)
    make_call(0, ref_a)()
    make_call(1, ref_b)()
    torch.cuda.synchronize()
    calls = [make_call(0, out_a), make_call(1, out_b)]
    s = [torch.cuda.Stream(), torch.cuda.Stream()]
    for _ in range(REPS):
        for k in (0, 1):
            with torch.cuda.stream(s[k]):
                calls[k]()
    torch.cuda.synchronize()
    assert torch.equal(out_a, ref_a)
    assert torch.equal(out_b, ref_b)


def _ws(pkv, b):
    return torch.empty(pkv.paged_attention_workspace_size(b.num_seqs, b.num_heads, b.num_kv_heads, b.head_dim,
                                                          b.block_size, b.max_context_len),
                       dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("name,path", [("llama13b_mixed_bs16", PATH_SIMT), ("long_trace", PATH_TENSOR),
                                       ("prefix_beams", PATH_TENSOR)])
def test_decode_on_two_streams(pkv, name, path):
    dbs = [DeviceBatch(wl.make_decode_batch(name, num_seqs=8, length_scale=0.15, seed=900 + k)) for k in (0, 1)]
    wss = [_ws(pkv, db.b) for db in dbs]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def make_call(k, out):
        db, ws = dbs[k], wss[k]
        return lambda: pkv.paged_attention_decode(out, db.query, db.key_cache, db.value_cache, db.tables, db.lens,
                                                  db.b.max_context_len, db.b.scale, ws, path=path, status=st)

    outs = [torch.empty((db.b.num_seqs, db.b.num_heads, db.b.head_dim), dtype=torch.float32, device="cuda")
            for db in dbs]
    _run_two_streams(make_call, *outs)
    assert st.item() == 0


def test_fp8_tensor_decode_on_two_streams(pkv):
    batches = [fp8_batch("long_trace", seed=910 + k, num_seqs=6, length_scale=0.15) for k in (0, 1)]
    dev = []
    for b, kc, vc, ks, vs in batches:
        dev.append((b, dev_bf16(b.query), u8(kc), u8(vc), f32(ks), f32(vs),
                    torch.from_numpy(np.ascontiguousarray(b.block_tables, np.int32)).cuda(),
                    torch.from_numpy(np.ascontiguousarray(b.context_lens, np.int32)).cuda(), _ws(pkv, b)))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def make_call(k, out):
        b, q, kc, vc, ks, vs, tables, lens, ws = dev[k]
        return lambda: pkv.paged_attention_decode_fp8(out, q, kc, vc, ks, vs, tables, lens, b.max_context_len,
                                                      b.scale, ws, path=PATH_TENSOR, status=st)

    outs = [torch.empty((d[0].num_seqs, d[0].num_heads, d[0].head_dim), dtype=torch.bfloat16, device="cuda")
            for d in dev]
    _run_two_streams(make_call, *outs)
    assert st.item() == 0


def test_prefill_on_two_streams(pkv):
    bs = [wl.make_prefill_batch("chunked_prefill_long_gqa", seed=920 + k, num_seqs=2, length_scale=0.05)
          for k in (0, 1)]
    dev = []
    for b in bs:
        ws = torch.empty(pkv.paged_attention_prefill_workspace_size(b.num_seqs, b.total_q, b.num_heads,
                                                                    b.num_kv_heads), dtype=torch.uint8, device="cuda")
        dev.append((b, dev_bf16(b.query), dev_bf16(b.key_cache), dev_bf16(b.value_cache),
                    torch.from_numpy(np.ascontiguousarray(b.block_tables, np.int32)).cuda(),
                    torch.from_numpy(np.ascontiguousarray(b.query_start, np.int32)).cuda(),
                    torch.from_numpy(np.ascontiguousarray(b.context_lens, np.int32)).cuda(), ws))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def make_call(k, out):
        b, q, kc, vc, tables, qstart, lens, ws = dev[k]
        return lambda: pkv.paged_attention_prefill(out, q, kc, vc, tables, qstart, lens, b.max_context_len, b.scale,
                                                   ws, status=st)

    outs = [torch.empty((d[0].total_q, d[0].num_heads, d[0].head_dim), dtype=torch.float32, device="cuda")
            for d in dev]
    _run_two_streams(make_call, *outs)
    assert st.item() == 0
