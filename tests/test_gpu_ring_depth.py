"""Race check for the CUDA-core decode kernel, where compute-sanitizer is not available.

The same decodes run through a build whose per-warp copy ring has one stage. There every copy
waits for the previous stage's compute, so no copy can land in a slot that is still being read.
The results must be bit-identical to the default two-stage build. Each item's accumulation
order depends neither on the ring depth nor on which warp runs the item, so any difference is
a pipelining race."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_one_stage_ring_matches_the_default_build(pkv, tmp_path):
    from paged_kv_cache_423_b200 import build as pkv_build
    from tests.ring_depth_cases import run_cases

    lib1 = pkv_build.build_library(variant="depth1")
    out_file = tmp_path / "depth1.npz"
    env = dict(os.environ, PKV_LIBRARY=lib1, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "ring_depth_cases.py"), str(out_file)],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    got = np.load(out_file)
    assert str(got["library"]) == lib1
    ref = run_cases(pkv)
    assert set(ref) == set(got.files) - {"library"}
    for name, v in ref.items():
        assert np.array_equal(v.view(np.uint32), got[name].view(np.uint32)), name
