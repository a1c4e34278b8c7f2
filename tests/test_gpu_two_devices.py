"""One process driving two GPUs: every launcher sets its kernel attributes up once per
device, so launches on cuda:0, then cuda:1, then cuda:0 again all run and match the
oracle.  Each device reads only its own memory.  Skipped where the process sees one GPU."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import fp8 as oracle_fp8
from oracle import paged_attention as oracle_decode
from oracle import prefill as oracle_prefill
from tests.gpu_helpers import DeviceBatch, compare
from tests.test_gpu_fp8 import fp8_batch, run_fp8
from tests.test_gpu_prefill import DevicePrefill

pytestmark = pytest.mark.gpu


@pytest.fixture
def two_devices():
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two GPUs visible to one process")
    return [0, 1, 0]


def test_decode_on_two_devices(pkv, two_devices):
    b = wl.make_decode_batch("prefix_beams", num_seqs=6, length_scale=0.2)
    ref = oracle_decode.paged_decode(b.query, b.key_cache, b.value_cache, b.block_tables, b.context_lens, b.scale)
    for dev in two_devices:
        with torch.cuda.device(dev):
            db = DeviceBatch(b)
            for path in (1, 2):      # CUDA cores, tensor cores
                out = db.decode(pkv, path=path)
                assert out.device.index == dev
                compare(out.cpu().numpy(), ref)


def test_prefill_on_two_devices(pkv, two_devices):
    b = wl.make_prefill_batch("chunked_prefill_13b", num_heads=8, num_kv_heads=2, query_lens=[33, 90, 1],
                              earlier_lens=[500, 31, 6])
    ref = oracle_prefill.paged_prefill(b.query, b.key_cache, b.value_cache, b.block_tables, b.query_start,
                                       b.context_lens, b.scale)
    for dev in two_devices:
        with torch.cuda.device(dev):
            compare(DevicePrefill(b).run(pkv).cpu().numpy(), ref)


def test_fp8_decode_on_two_devices(pkv, two_devices):
    b, kc, vc, ks, vs = fp8_batch("long_trace", num_seqs=2, length_scale=0.05)
    ref = oracle_fp8.paged_decode_fp8(b.query, kc, vc, ks, vs, b.block_tables, b.context_lens, b.scale)
    for dev in two_devices:
        with torch.cuda.device(dev):
            for path in (1, 2):
                compare(run_fp8(pkv, b, kc, vc, ks, vs, path=path).cpu().numpy(), ref)
