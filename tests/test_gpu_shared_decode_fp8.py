"""Shared-prefix decode over 8-bit (e4m3) pools (pkv_paged_attention_decode_shared_fp8) on the
GPU against the float64 8-bit oracle: the result must be that of plain decode attention over
each row's whole context on the dequantised pool (Outcome School explainer, "内存共享": rows
share blocks, not results; intelliparadigm article §4.2, §5: fp8 KV).  The pools are drawn as
e4m3 bit patterns with per-kv-head scales, as for the 8-bit decode tests.  Batches: a shared
system prompt (small, and full size on sampled rows), beam forks with copy-on-write after
appends (nested segments), several key-chunk sizes, block size 32, a batch with no sharing, a
plan that no longer fits the lengths (flagged, zero output), a plan whose scratch blocks run
past the scratch pools (flagged, zero output) and a shared block outside the pool (flagged).
Tolerance as for decode (fp32 output)."""
import numpy as np
import pytest
import torch

import workloads as wl
from oracle import fp8 as oracle
from tests.gpu_helpers import compare, dev_bf16
from tests.test_gpu_fp8 import f32, u8
from tests.test_gpu_shared_decode import beam_batch

pytestmark = pytest.mark.gpu


class Pool8:
    """A batch's tables and lengths with e4m3 pools and per-kv-head scales on the GPU."""

    def __init__(self, b, seed):
        rng = wl.rng_for(seed)
        self.b = b
        shape = (b.num_blocks, b.num_kv_heads, b.block_size, b.head_dim)
        self.kc, self.vc = wl.e4m3_codes(rng, shape), wl.e4m3_codes(rng, shape)
        self.ks, self.vs = wl.kv_scales(rng, b.num_kv_heads), wl.kv_scales(rng, b.num_kv_heads)
        self.query = dev_bf16(b.query)
        self.kc_d, self.vc_d, self.ks_d, self.vs_d = u8(self.kc), u8(self.vc), f32(self.ks), f32(self.vs)
        self.tables = torch.from_numpy(np.ascontiguousarray(b.block_tables, np.int32)).cuda()
        self.lens = torch.from_numpy(np.ascontiguousarray(b.context_lens, np.int32)).cuda()

    def oracle(self, rows=None):
        b = self.b
        rows = list(range(b.num_seqs) if rows is None else rows)
        return oracle.paged_decode_fp8(b.query[rows], self.kc, self.vc, self.ks, self.vs,
                                       np.asarray(b.block_tables)[rows], np.asarray(b.context_lens)[rows], b.scale)


def run_shared(pkv, p, key_chunk=0, out_dtype=torch.float32, lens=None, plan_tables=None, status=None, min_rows=2):
    b = p.b
    tables_h = b.block_tables if plan_tables is None else plan_tables
    plan, info = pkv.shared_plan(tables_h, b.context_lens, b.num_heads, b.num_kv_heads, b.block_size,
                                 min_rows=min_rows, key_chunk=key_chunk)
    plan_d = torch.from_numpy(plan).cuda()
    ws = torch.empty(pkv.paged_attention_decode_shared_fp8_workspace_size(info, b.num_heads, b.num_kv_heads,
                                                                          b.head_dim),
                     dtype=torch.uint8, device="cuda")
    out = torch.full((b.num_seqs, b.num_heads, b.head_dim), float("nan"), dtype=out_dtype, device="cuda")
    own = status is None
    if own:
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tables = p.tables if plan_tables is None else torch.from_numpy(np.ascontiguousarray(plan_tables, np.int32)).cuda()
    pkv.paged_attention_decode_shared_fp8(out, p.query, p.kc_d, p.vc_d, p.ks_d, p.vs_d, tables,
                                          p.lens if lens is None else lens, b.scale, plan_d, info, ws, status=status)
    torch.cuda.synchronize()
    if own:
        assert status.item() == 0, f"device status {status.item():#x}"
    return out, info


@pytest.mark.parametrize("key_chunk", [0, 128, 256])
def test_shared_prompt_matches_oracle(pkv, key_chunk):
    p = Pool8(wl.make_decode_batch("prefix_beams", num_seqs=12, length_scale=0.3), 1200)
    out, info = run_shared(pkv, p, key_chunk=key_chunk)
    assert info.num_segments == 1 and info.num_partials > 0
    compare(out.cpu().numpy(), p.oracle())


@pytest.mark.parametrize("steps", [0, 1, 3])
@pytest.mark.parametrize("heads", [(32, 8), (16, 8), (64, 4)])
def test_beam_forks_match_oracle(pkv, steps, heads):
    p = Pool8(beam_batch(70 + steps, steps=steps, Hq=heads[0], Hkv=heads[1]), 1210 + steps)
    out, info = run_shared(pkv, p)
    assert info.num_segments >= 1
    compare(out.cpu().numpy(), p.oracle())


@pytest.mark.parametrize("steps", [1, 3])
def test_beam_forks_without_beam_segments(pkv, steps):
    """Segments of at least 5 rows only (the choice for 8-bit pools): the beams' parent blocks
    stay in their private remainders, read by the 8-bit decode; the result is the same."""
    p = Pool8(beam_batch(75 + steps, steps=steps), 1215 + steps)
    out, info = run_shared(pkv, p, min_rows=5)
    compare(out.cpu().numpy(), p.oracle())


def test_block_size_32(pkv):
    p = Pool8(beam_batch(81, bs=32, prompt_tokens=320, steps=2), 1220)
    out, _ = run_shared(pkv, p)
    compare(out.cpu().numpy(), p.oracle())


def test_bf16_output_is_the_rounded_f32_output(pkv):
    p = Pool8(beam_batch(82, steps=1), 1230)
    f32_out, _ = run_shared(pkv, p)
    bf16_out, _ = run_shared(pkv, p, out_dtype=torch.bfloat16)
    assert torch.equal(bf16_out, f32_out.to(torch.bfloat16))


def test_no_sharing_equals_decode(pkv):
    p = Pool8(wl.make_decode_batch("long_trace", num_seqs=3, length_scale=0.06), 1240)
    out, info = run_shared(pkv, p)
    assert info.num_segments == 0
    compare(out.cpu().numpy(), p.oracle())


def test_full_size_shared_prompt_sampled(pkv):
    """The 128-sequence shared-prompt batch (1024-token prompt), sampled rows against the oracle."""
    b = wl.make_decode_batch("prefix_beams", with_data=False)
    b.query = wl.bf16_normal(wl.rng_for(1250), (b.num_seqs, b.num_heads, b.head_dim))
    p = Pool8(b, 1251)
    out, info = run_shared(pkv, p)
    assert info.num_segments == 1 and info.shared_tokens == wl.PREFIX_TOKENS
    rows = sorted(wl.rng_for(1252).choice(b.num_seqs, 6, replace=False).tolist())
    compare(out.cpu().numpy()[rows], p.oracle(rows))


def test_stale_plan_is_flagged_and_zeroed(pkv):
    p = Pool8(beam_batch(83, steps=1), 1260)
    lens = p.b.context_lens.copy()
    lens[2] += 1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, _ = run_shared(pkv, p, lens=torch.from_numpy(lens).cuda(), status=status)
    assert status.item() & pkv.PKV_DEV_BAD_CONTEXT
    assert torch.all(out == 0)
    out, _ = run_shared(pkv, p)  # the same plan and pools work again with the right lengths
    compare(out.cpu().numpy(), p.oracle())


def test_shared_block_outside_the_pool_is_flagged(pkv):
    """A shared block id past the pool in every row that shares it: PKV_DEV_BAD_BLOCK, nothing
    read out of range, every output finite."""
    p = Pool8(wl.make_decode_batch("prefix_beams", num_seqs=8, length_scale=0.3), 1270)
    tables = np.array(p.b.block_tables, np.int32, copy=True)
    tables[:, 3] = p.b.num_blocks + 5  # the prompt's fourth block, in every table
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, info = run_shared(pkv, p, plan_tables=tables, status=status)
    assert info.num_segments == 1
    assert status.item() & pkv.PKV_DEV_BAD_BLOCK
    assert torch.isfinite(out).all()


def test_plan_with_a_bad_scratch_base_is_flagged_and_zeroed(pkv):
    """A part whose scratch blocks would run past the scratch pools: the plan check rejects the
    plan (PKV_DEV_BAD_CONTEXT, zero rows) before anything is widened or read."""
    p = Pool8(wl.make_decode_batch("prefix_beams", num_seqs=8, length_scale=0.3), 1280)
    b = p.b
    plan, info = pkv.shared_plan(b.block_tables, b.context_lens, b.num_heads, b.num_kv_heads, b.block_size)
    words = plan.view(np.int32)
    words[info.off_parts // 4 + 6] = 1 << 20  # part 0's first scratch block
    ws = torch.empty(pkv.paged_attention_decode_shared_fp8_workspace_size(info, b.num_heads, b.num_kv_heads,
                                                                          b.head_dim), dtype=torch.uint8, device="cuda")
    out = torch.full((b.num_seqs, b.num_heads, b.head_dim), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_attention_decode_shared_fp8(out, p.query, p.kc_d, p.vc_d, p.ks_d, p.vs_d, p.tables, p.lens, b.scale,
                                          torch.from_numpy(plan).cuda(), info, ws, status=status)
    torch.cuda.synchronize()
    assert status.item() & pkv.PKV_DEV_BAD_CONTEXT
    assert torch.all(out == 0)


def test_long_remainders_match_oracle(pkv):
    """Private remainders past one 128-token tile go through the 8-bit tensor-core decode (shorter
    ones through the 8-bit CUDA-core decode, as in the beam batches here): a shared prompt with long
    remainders."""
    lens = 1024 + np.array([1100, 1350, 1600, 1200, 1500], np.int32)
    p = Pool8(wl.make_decode_batch("prefix_beams", lengths=lens, seed=92), 1290)
    out, info = run_shared(pkv, p)
    assert info.num_segments == 1 and info.max_suffix_len > 1024
    compare(out.cpu().numpy(), p.oracle())
