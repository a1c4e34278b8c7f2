"""The launches of the bounded-wait expiry test.

Run as a script with PKV_LIBRARY naming the short-wait build (its CUDA-core decode and
prefill kernels give up a pipeline wait after one poll), it runs a small
decode (CUDA-core path, unsplit and split) and a small chunked prefill through that build
and records each call's device status word; then, in the same process and CUDA context,
it loads the default build named by its second argument and runs the same decode and
prefill again.  It writes the statuses and the default build's outputs to the .npz file
named by its first argument."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def batches():
    import workloads as wl
    d = wl.make_decode_batch("llama7b", num_seqs=6, length_scale=0.3, num_heads=8, num_kv_heads=8)
    p = wl.make_prefill_batch("chunked_prefill_13b", num_heads=8, num_kv_heads=2, query_lens=[33, 200, 1],
                              earlier_lens=[500, 31, 6])
    return d, p


def run(pkv, d, p):
    import torch

    from tests.gpu_helpers import DeviceBatch
    from tests.test_gpu_prefill import DevicePrefill
    res = {}
    db = DeviceBatch(d)
    for part in (0, 64):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        res[f"decode_p{part}"] = (db.decode(pkv, partition=part, path=pkv.PATH_SIMT, status=st).cpu().numpy(),
                                  int(st.item()))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    res["prefill"] = (DevicePrefill(p).run(pkv, status=st).cpu().numpy(), int(st.item()))
    return res


if __name__ == "__main__":
    import torch

    import paged_kv_cache_423_b200 as pkv
    d, p = batches()
    short_lib = pkv.library_path()
    short = run(pkv, d, p)
    torch.cuda.synchronize()
    # the default build, loaded into the same process and context
    os.environ["PKV_LIBRARY"] = sys.argv[2]
    pkv._lib = None
    assert pkv.library_path() == sys.argv[2]
    default = run(pkv, d, p)
    out = {"short_library": np.array(short_lib), "default_library": np.array(pkv.library_path())}
    for k, (_, st) in short.items():
        out[f"{k}_short_status"] = np.array(st)
    for k, (o, st) in default.items():
        out[f"{k}_out"] = o
        out[f"{k}_status"] = np.array(st)
    np.savez(sys.argv[1], **out)
