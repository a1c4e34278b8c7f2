"""Helpers of the GPU parity tests: move seeded inputs to the device, call the
library through its binding, and compare against the oracle."""
import numpy as np
import torch

# Attention tolerance against the float64 oracle (bf16 inputs, fp32 accumulation).
MAX_ABS_TOL = 1e-2
REL_L2_TOL = 5e-3


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def compare(got: np.ndarray, ref: np.ndarray, max_abs=MAX_ABS_TOL, rel_l2=REL_L2_TOL):
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref)
    ma = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rl2 = float(np.linalg.norm(got - ref) / denom) if denom > 0 else float(np.linalg.norm(got - ref))
    assert np.all(np.isfinite(got)), "non-finite output"
    assert ma <= max_abs, f"max-abs error {ma:.3e} > {max_abs:.1e}"
    assert rl2 <= rel_l2, f"relative-L2 error {rl2:.3e} > {rel_l2:.1e}"
    return ma, rl2


class DeviceBatch:
    """A workloads.DecodeBatch resident on the GPU."""

    def __init__(self, batch, key_cache=None, value_cache=None):
        self.b = batch
        self.query = dev_bf16(batch.query)
        self.key_cache = key_cache if key_cache is not None else dev_bf16(batch.key_cache)
        self.value_cache = value_cache if value_cache is not None else dev_bf16(batch.value_cache)
        self.tables = torch.from_numpy(np.ascontiguousarray(batch.block_tables, np.int32)).cuda()
        self.lens = torch.from_numpy(np.ascontiguousarray(batch.context_lens, np.int32)).cuda()

    def decode(self, pkv, out_dtype=torch.float32, partition=0, path=0, max_context_len=None, status=None):
        b = self.b
        maxl = b.max_context_len if max_context_len is None else max_context_len
        ws_bytes = pkv.paged_attention_workspace_size(b.num_seqs, b.num_heads, b.num_kv_heads, b.head_dim,
                                                      b.block_size, maxl, partition)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        out = torch.empty((b.num_seqs, b.num_heads, b.head_dim), dtype=out_dtype, device="cuda")
        own_status = status is None
        if own_status:
            status = torch.zeros(1, dtype=torch.int32, device="cuda")
        pkv.paged_attention_decode(out, self.query, self.key_cache, self.value_cache, self.tables, self.lens, maxl,
                                   b.scale, ws, partition_tokens=partition, path=path, status=status)
        torch.cuda.synchronize()
        if own_status:
            assert status.item() == 0, f"device status {status.item():#x}"
        return out
