"""Decode without a caller-provided workspace.

Some users of this library cannot allocate device memory: a plugin called through
a host runtime's custom-operator interface may receive only its input and output
buffers, and some applications give all device memory to their own allocator or
forbid allocations while they run.  pkv_paged_attention_decode_static serves them
with scratch built into the library.  These tests call it through the C ABI and
check it against pkv_paged_attention_decode (which takes a workspace) on two
calls in a row, with batches whose long sequences are split into partitions, so
the built-in scratch really holds partials and counters left over from the call
before.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl
from tests.gpu_helpers import MAX_ABS_TOL, REL_L2_TOL, DeviceBatch, compare


def _call_static(lib, db, out, partition):
    b = db.b
    return lib.pkv_paged_attention_decode_static(
        out.data_ptr(), 1, db.query.data_ptr(), db.key_cache.data_ptr(), db.value_cache.data_ptr(),
        db.tables.data_ptr(), db.tables.shape[1], db.lens.data_ptr(), b.max_context_len, b.num_seqs, b.num_heads,
        b.num_kv_heads, b.head_dim, b.block_size, b.num_blocks, b.scale, partition, 0, None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_point(pkv):
    lib = pkv.library()
    batches = [
        wl.make_decode_batch("llama7b", num_seqs=6, num_heads=8, num_kv_heads=8, lengths=[1, 63, 700, 1500, 2000, 17]),
        wl.make_decode_batch("long_trace", num_seqs=3, length_scale=0.1),
    ]
    for b, partition in zip(batches, (128, 64)):
        db = DeviceBatch(b)
        ref = db.decode(pkv, out_dtype=torch.float32, partition=partition)
        out = torch.full_like(ref, float("nan"))
        rc = _call_static(lib, db, out, partition)
        assert rc == pkv.PKV_OK, lib.pkv_last_error_string().decode()
        torch.cuda.synchronize()
        compare(out.cpu().numpy(), ref.cpu().numpy().astype(np.float64), MAX_ABS_TOL, REL_L2_TOL)


def test_static_scratch_rejects_work_beyond_its_size(pkv):
    lib = pkv.library()
    fake = ctypes.c_void_p(0x1000)
    need = lib.pkv_paged_attention_workspace_size(4096, 64, 8, 128, 32, 32768, 0)
    assert need > pkv.STATIC_SCRATCH_BYTES
    rc = lib.pkv_paged_attention_decode_static(fake, 1, fake, fake, fake, fake, 1024, fake, 32768, 4096, 64, 8, 128,
                                               32, 100000, 0.1, 0, 0, None, None)
    assert rc == pkv.PKV_ERR_INVALID
    assert b"built-in array" in lib.pkv_last_error_string()
