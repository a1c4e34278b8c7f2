"""Decode calls captured in a CUDA graph and replayed.

A call launches its plan, the decode kernel and, on the tensor-core paths, the split merge
(and the query split of the 8-bit path) back to back, each later kernel launched to start
while the one before it finishes.  Captured once and replayed, the call must give the same
bytes as the direct call, and a replay after the query is rewritten in place must give what
a direct call on the new query gives: the graph holds pointers, not values."""
import numpy as np
import pytest
import torch

import workloads as wl
from tests.gpu_helpers import DeviceBatch, dev_bf16
from tests.test_gpu_fp8 import f32, fp8_batch, u8

pytestmark = pytest.mark.gpu

PATH_SIMT, PATH_TENSOR = 1, 2


def _replay_matches(call, query, out):
    """call(out) decodes into `out`; compare direct, captured and replayed results."""
    direct = torch.empty_like(out)
    call(direct)                                   # also sets up the kernels before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(out)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, direct)
    # new query values in the same buffer
    query.copy_(torch.flip(query, dims=[0]))
    call(direct)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, direct)


@pytest.mark.parametrize("name,path", [("llama13b_mixed_bs16", PATH_SIMT), ("long_trace", PATH_TENSOR),
                                       ("prefix_beams", PATH_TENSOR)])
def test_bf16_decode_replays(pkv, name, path):
    b = wl.make_decode_batch(name, num_seqs=6, length_scale=0.1)
    db = DeviceBatch(b)
    ws = torch.empty(pkv.paged_attention_workspace_size(b.num_seqs, b.num_heads, b.num_kv_heads, b.head_dim,
                                                        b.block_size, b.max_context_len),
                     dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty((b.num_seqs, b.num_heads, b.head_dim), dtype=torch.float32, device="cuda")

    def call(o):
        pkv.paged_attention_decode(o, db.query, db.key_cache, db.value_cache, db.tables, db.lens, b.max_context_len,
                                   b.scale, ws, path=path, status=status)

    _replay_matches(call, db.query, out)
    assert status.item() == 0


def test_fp8_tensor_decode_replays(pkv):
    b, kc, vc, ks, vs = fp8_batch("long_trace", num_seqs=4, length_scale=0.1)
    q = dev_bf16(b.query)
    kc_d, vc_d, ks_d, vs_d = u8(kc), u8(vc), f32(ks), f32(vs)
    tables = torch.from_numpy(np.ascontiguousarray(b.block_tables, np.int32)).cuda()
    lens = torch.from_numpy(np.ascontiguousarray(b.context_lens, np.int32)).cuda()
    ws = torch.empty(pkv.paged_attention_workspace_size(b.num_seqs, b.num_heads, b.num_kv_heads, b.head_dim,
                                                        b.block_size, b.max_context_len),
                     dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty((b.num_seqs, b.num_heads, b.head_dim), dtype=torch.bfloat16, device="cuda")

    def call(o):
        pkv.paged_attention_decode_fp8(o, q, kc_d, vc_d, ks_d, vs_d, tables, lens, b.max_context_len, b.scale, ws,
                                       path=PATH_TENSOR, status=status)

    _replay_matches(call, q, out)
    assert status.item() == 0
