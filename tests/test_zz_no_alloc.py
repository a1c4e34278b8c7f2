"""Decode without a caller-provided workspace.

Some users of this library cannot allocate device memory: a plugin called through
a host runtime's custom-operator interface may receive only its input and output
buffers, and some applications give all device memory to their own allocator or
forbid allocations while they run.  pkv_paged_attention_decode_static serves them
with scratch built into the library.  These tests call it through the C ABI and
check it against pkv_paged_attention_decode (which takes a workspace) on two
calls in a row, with batches whose long sequences are split into partitions, so
the built-in scratch really holds partials and counters left over from the call
before.  Both entry points run the same plan and kernels, so their outputs must be
bit-identical; a device status word is passed and checked on every call.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import workloads as wl
from oracle import paged_attention as oracle
from tests.gpu_helpers import DeviceBatch, compare


def _call_static(lib, db, out, partition, status, path=0):
    b = db.b
    return lib.pkv_paged_attention_decode_static(
        out.data_ptr(), 1 if out.dtype == torch.float32 else 0, db.query.data_ptr(), db.key_cache.data_ptr(),
        db.value_cache.data_ptr(), db.tables.data_ptr(), db.tables.shape[1], db.lens.data_ptr(), b.max_context_len,
        b.num_seqs, b.num_heads, b.num_kv_heads, b.head_dim, b.block_size, b.num_blocks, b.scale, partition, path,
        ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


BATCHES = {
    # long sequences split into partitions of 128 tokens: partials and counters live in the scratch
    "mha_split": (dict(name="llama7b", num_seqs=6, num_heads=8, num_kv_heads=8,
                       lengths=[1, 63, 700, 1500, 2000, 17]), 128, 0),
    # grouped heads on the tensor cores, split into 64-token partitions
    "gqa_split": (dict(name="long_trace", num_seqs=3, length_scale=0.1), 64, 0),
    # the same grouped batch on the CUDA cores
    "gqa_split_simt": (dict(name="long_trace", num_seqs=3, length_scale=0.1), 256, 1),
}


@pytest.mark.gpu
@pytest.mark.parametrize("case", sorted(BATCHES))
def test_static_scratch_matches_workspace_entry_point(pkv, case):
    """Two calls in a row (the second sees the first one's scratch) give exactly the
    output of the workspace entry point, with a clean status word."""
    lib = pkv.library()
    kw, partition, path = BATCHES[case]
    db = DeviceBatch(wl.make_decode_batch(**kw))
    ref = db.decode(pkv, out_dtype=torch.float32, partition=partition, path=path)
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = _call_static(lib, db, out, partition, status, path)
        assert rc == pkv.PKV_OK, lib.pkv_last_error_string().decode()
        torch.cuda.synchronize()
        assert status.item() == 0, f"device status {status.item():#x}"
        assert torch.equal(out, ref), "static-scratch output differs from the workspace entry point"


@pytest.mark.gpu
def test_static_scratch_matches_the_oracle(pkv):
    """The static entry point on its own against the float64 oracle, through the Python
    wrapper (bf16 output is checked against the f32 call's rounding elsewhere; here f32)."""
    b = wl.make_decode_batch("prefix_beams", num_seqs=10, length_scale=0.3)
    db = DeviceBatch(b)
    ref = oracle.paged_decode(b.query, b.key_cache, b.value_cache, b.block_tables, b.context_lens, b.scale)
    for partition in (0, 128):
        out = torch.full((b.num_seqs, b.num_heads, b.head_dim), float("nan"), dtype=torch.float32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        pkv.paged_attention_decode_static(out, db.query, db.key_cache, db.value_cache, db.tables, db.lens,
                                          b.max_context_len, b.scale, partition_tokens=partition, status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        compare(out.cpu().numpy(), ref)


def test_static_scratch_rejects_work_beyond_its_size(pkv):
    lib = pkv.library()
    fake = ctypes.c_void_p(0x1000)
    need = lib.pkv_paged_attention_workspace_size(4096, 64, 8, 128, 32, 32768, 0)
    assert need > pkv.STATIC_SCRATCH_BYTES
    rc = lib.pkv_paged_attention_decode_static(fake, 1, fake, fake, fake, fake, 1024, fake, 32768, 4096, 64, 8, 128,
                                               32, 100000, 0.1, 0, 0, None, None)
    assert rc == pkv.PKV_ERR_INVALID
    assert b"built-in array" in lib.pkv_last_error_string()


@pytest.mark.parametrize("head_dim,block_size,path", [(128, 8, 0), (96, 16, 0), (64, 16, 2), (128, 16, 7)])
def test_static_scratch_refuses_what_the_workspace_variant_refuses(pkv, head_dim, block_size, path):
    """Unsupported sizes give the workspace variant's return code, with nothing launched
    (the pointers are fake: a launch would be an error of its own)."""
    lib = pkv.library()
    fake = ctypes.c_void_p(0x1000)
    args = (fake, 1, fake, fake, fake, fake, 64, fake, 1000, 4, 8, 2, head_dim, block_size, 1000, 0.1, 0, path)
    rc_static = lib.pkv_paged_attention_decode_static(*args, None, None)
    rc_ws = lib.pkv_paged_attention_decode(*args, fake, 1 << 20, None, None)
    assert rc_static == rc_ws and rc_ws in (pkv.PKV_ERR_UNSUPPORTED, pkv.PKV_ERR_INVALID)


def test_static_scratch_size_matches_the_header(pkv):
    """The binding's STATIC_SCRATCH_BYTES is the header's PKV_STATIC_SCRATCH_BYTES."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "include", "pkv.h")) as f:
        m = re.search(r"#define PKV_STATIC_SCRATCH_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", f.read())
    assert m is not None
    assert pkv.STATIC_SCRATCH_BYTES == int(m.group(1)) * int(m.group(2)) * int(m.group(3))
