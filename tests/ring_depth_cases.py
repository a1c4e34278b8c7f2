"""The CUDA-core decodes a ring-depth comparison runs.

`run_cases(pkv)` builds its seeded inputs the same way in every process and returns
the float32 outputs by name: bf16 pools (one head per kv head, and four), 8-bit pools,
each unsplit and split into 64-token partitions, all on the CUDA-core path.  Run as a
script it loads the library the binding resolves (PKV_LIBRARY, if set) and writes the
outputs, with that library's path, to the .npz file named by its argument."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def run_cases(pkv):
    import torch

    import workloads as wl
    from tests.gpu_helpers import DeviceBatch, dev_bf16

    outs = {}
    for name, kw in (("mha", dict(num_seqs=8, length_scale=0.3)),
                     ("gqa4", dict(num_seqs=6, length_scale=0.3, num_heads=8, num_kv_heads=2))):
        db = DeviceBatch(wl.make_decode_batch("llama7b", **kw))
        for part in (0, 64):
            outs[f"{name}_p{part}"] = db.decode(pkv, partition=part, path=pkv.PATH_SIMT).cpu().numpy()
    b = wl.make_decode_batch("llama7b", with_data=False, num_seqs=8, length_scale=0.3)
    rng = wl.rng_for(830)
    q = wl.bf16_normal(rng, (b.num_seqs, b.num_heads, b.head_dim))
    shape = (b.num_blocks, b.num_kv_heads, b.block_size, b.head_dim)
    kc = torch.from_numpy(wl.e4m3_codes(rng, shape)).cuda()
    vc = torch.from_numpy(wl.e4m3_codes(rng, shape)).cuda()
    ks = torch.from_numpy(wl.kv_scales(rng, b.num_kv_heads)).cuda()
    vs = torch.from_numpy(wl.kv_scales(rng, b.num_kv_heads)).cuda()
    tables = torch.from_numpy(np.ascontiguousarray(b.block_tables, np.int32)).cuda()
    lens = torch.from_numpy(np.ascontiguousarray(b.context_lens, np.int32)).cuda()
    for part in (0, 64):
        ws = torch.empty(pkv.paged_attention_workspace_size(b.num_seqs, b.num_heads, b.num_kv_heads, b.head_dim,
                                                            b.block_size, b.max_context_len, part),
                         dtype=torch.uint8, device="cuda")
        out = torch.empty((b.num_seqs, b.num_heads, b.head_dim), dtype=torch.float32, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        pkv.paged_attention_decode_fp8(out, dev_bf16(q), kc, vc, ks, vs, tables, lens, b.max_context_len, b.scale, ws,
                                       partition_tokens=part, path=pkv.PATH_SIMT, status=status)
        torch.cuda.synchronize()
        assert status.item() == 0, f"device status {status.item():#x}"
        outs[f"kv8_p{part}"] = out.cpu().numpy()
    return outs


if __name__ == "__main__":
    import paged_kv_cache_423_b200 as pkv
    results = run_cases(pkv)
    np.savez(sys.argv[1], library=np.array(pkv.library_path()), **results)
