"""The expiry path of the bounded on-chip waits, made to run on an ordinary launch.

Every mbarrier wait of the kernels gives up after a limit (one second of %globaltimer)
and the kernel then flags PKV_DEV_TIMEOUT, lets its copies in flight land, waits for its
MMAs, frees its tensor memory and returns, so a scheduling bug cannot hang the GPU.  A
second build of the library (`build_library(variant="shortwait")`) shortens the pipeline
waits of the CUDA-core decode and of the prefill kernel to a single poll -- no wait is
removed, and the end-of-kernel drains keep their full limit -- so ordinary decode and
prefill launches run into that path.  In a child process the test
requires (1) every short-wait call to return with PKV_DEV_TIMEOUT in its status word and
(2) the default build, loaded afterwards into the same process and CUDA context, to give
the oracle's results with a clean status: the context stays usable."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_short_waits_time_out_and_the_context_stays_usable(pkv, tmp_path):
    from oracle import paged_attention, prefill
    from paged_kv_cache_423_b200 import build as pkv_build
    from tests.gpu_helpers import compare
    from tests.timeout_cases import batches

    short_lib = pkv_build.build_library(variant="shortwait")
    default_lib = pkv_build.build_library()
    out_file = tmp_path / "timeout.npz"
    env = dict(os.environ, PKV_LIBRARY=short_lib, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "timeout_cases.py"), str(out_file), default_lib],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    got = np.load(out_file)
    assert str(got["short_library"]) == short_lib and str(got["default_library"]) == default_lib
    for k in ("decode_p0", "decode_p64", "prefill"):
        assert int(got[f"{k}_short_status"]) & pkv.PKV_DEV_TIMEOUT, k
        assert int(got[f"{k}_status"]) == 0, k
    d, p = batches()
    ref = paged_attention.paged_decode(d.query, d.key_cache, d.value_cache, d.block_tables, d.context_lens, d.scale)
    compare(got["decode_p0_out"], ref)
    compare(got["decode_p64_out"], ref)
    ref_p = prefill.paged_prefill(p.query, p.key_cache, p.value_cache, p.block_tables, p.query_start, p.context_lens,
                                  p.scale)
    compare(got["prefill_out"], ref_p)
