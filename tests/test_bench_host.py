"""Host-side logic of bench.py: byte accounting and the multi-rank aggregation
(world size 2 over gloo on CPU; the GPU runs use the same calls over NCCL)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def test_decode_bytes_counts_each_token_once():
    kv, alg = bench.decode_bytes([1, 16, 17], Hq=8, Hkv=2, D=128, bs=16)
    assert kv == 34 * 2 * 128 * 2 * 2
    blocks = 1 + 1 + 2
    assert alg == kv + 2 * 3 * 8 * 128 * 2 + blocks * 4 + 3 * 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms, units = bench.aggregate_over_ranks(10.0 + 5 * rank, 100 * (rank + 1), dist, torch.device("cpu"))
    results[rank] = (ms, units)
    dist.barrier()
    dist.destroy_process_group()


def test_aggregate_over_two_gloo_ranks():
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    # every rank sees the slowest rank's time and the units of all ranks
    assert results[0] == results[1] == (15.0, 300)


def test_single_process_aggregation_is_identity():
    assert bench.aggregate_over_ranks(3.5, 7) == (3.5, 7)


def test_prefill_flops_counts_every_visible_key():
    """4 * D FLOPs per (query row, head, visible key): the closed form against a
    brute-force count of the causal window of every row."""
    import bench
    qlens = np.array([3, 0, 7, 1])
    lens = np.array([10, 4, 7, 1])
    brute = 0
    for n, L in zip(qlens, lens):
        for i in range(n):
            brute += (L - n + i) + 1
    assert bench.prefill_flops(qlens, lens, 5, 128) == 4 * 128 * 5 * brute


def test_split_tokens_mirrors_the_library():
    """bench.split_tokens counts the merge launch of a split context; on the CUDA-core
    path it must be the library's own automatic split, and the tensor-core split is
    never shorter than it and at most 2048 tokens."""
    import paged_kv_cache_423_b200 as pkv
    for B in (1, 3, 16, 128, 256):
        for hkv in (1, 8, 40):
            for bs in (16, 32):
                for L in (1, 100, 2049, 32768, 131072):
                    simt = bench.split_tokens(B, hkv, bs, L, False)
                    assert simt == pkv.paged_attention_partition_tokens(B, hkv, bs, L)
                    tensor = bench.split_tokens(B, hkv, bs, L, True)
                    assert simt <= tensor <= 2048 and tensor % bs == 0


def test_all_cores_oracle_counts_every_sequence():
    """The all-cores oracle leg (spawned workers) processes every sampled sequence once per pass."""
    import types
    import workloads as wl
    b = wl.make_decode_batch("tiny")
    w = types.SimpleNamespace(Hkv=b.num_kv_heads, D=b.head_dim, scale=b.scale)
    items = []
    for s in range(b.num_seqs):
        need = -(-int(b.context_lens[s]) // b.block_size)
        blocks = b.block_tables[s][:need]
        items.append((b.query[s:s + 1], b.key_cache[blocks], b.value_cache[blocks],
                      np.arange(need, dtype=np.int32)[None, :], b.context_lens[s:s + 1]))
    done, dt, cores = bench.time_oracle_all_cores(w, items)
    assert done == cores * int(b.context_lens.sum()) * b.num_kv_heads * b.head_dim * 4  # `cores` passes
    assert cores >= 1 and dt > 0


def test_fp8_oracle_timer_counts_one_byte_per_value():
    """The 8-bit oracle timer (CPU-baseline leg and reference arm) counts K and V at 1 B each."""
    import types
    import workloads as wl
    b = wl.make_decode_batch("llama7b", num_seqs=3, num_heads=4, num_kv_heads=2, length_scale=0.02, with_data=False)
    rng = wl.rng_for(3)
    shape = (b.num_blocks, b.num_kv_heads, b.block_size, b.head_dim)
    kc, vc = wl.e4m3_codes(rng, shape), wl.e4m3_codes(rng, shape)
    ks, vs = wl.kv_scales(rng, b.num_kv_heads), wl.kv_scales(rng, b.num_kv_heads)
    q = wl.bf16_normal(rng, (b.num_seqs, b.num_heads, b.head_dim))
    w = types.SimpleNamespace(Hkv=b.num_kv_heads, D=b.head_dim, scale=b.scale)
    items = [(q[s:s + 1], kc, vc, ks, vs, b.block_tables[s:s + 1], b.context_lens[s:s + 1]) for s in range(b.num_seqs)]
    done, dt, n = bench.time_oracle_fp8(w, items, 60.0)
    assert n == b.num_seqs and dt > 0                      # one pass (the reference arm's timing)
    assert done == int(b.context_lens.sum()) * b.num_kv_heads * b.head_dim * 2
    done, dt, n = bench.time_oracle_fp8(w, items, 0.3, repeat=True)
    assert n > b.num_seqs and dt >= 0.3                    # passes until the budget (the CPU-baseline leg)
    per = [int(l) * b.num_kv_heads * b.head_dim * 2 for l in b.context_lens]
    assert done == sum(per[i % b.num_seqs] for i in range(n))


def _distinct_slots(tables, lens, bs):
    return len({int(tables[s][t // bs]) * bs + t % bs for s, L in enumerate(lens) for t in range(L)})


def test_unique_kv_bytes_counts_each_physical_slot_once():
    per_slot = 2 * 128 * 2 * 2  # Hkv=2, D=128, K and V, bf16
    # two sequences share block 7 (a full prefix block), then go their own ways; the
    # shorter one also reads a partial block; block 0 (padding) is past every length
    tables = np.array([[7, 3, 0], [7, 5, 9]], np.int32)
    lens = [20, 37]
    u = bench.unique_kv_bytes(tables, lens, Hkv=2, D=128, bs=16)
    assert u == _distinct_slots(tables, lens, 16) * per_slot == (16 + 4 + 16 + 5) * per_slot
    kv, _ = bench.decode_bytes(lens, Hq=8, Hkv=2, D=128, bs=16)
    assert kv - u == 16 * per_slot  # the shared block is the only difference
    # nothing shared: the same as the logical count; e4m3 halves it
    tables = np.array([[1, 2], [3, 4], [5, 0]], np.int32)
    lens = [32, 17, 0]
    assert bench.unique_kv_bytes(tables, lens, 2, 128, 16) == bench.decode_bytes(lens, 8, 2, 128, 16)[0]
    assert bench.unique_kv_bytes(tables, lens, 2, 128, 16, 1) * 2 == bench.decode_bytes(lens, 8, 2, 128, 16)[0]


def test_unique_kv_bytes_on_random_forked_tables():
    rng = np.random.default_rng(5)
    bs = 8
    for _ in range(20):
        n_shared = int(rng.integers(0, 4))
        B = int(rng.integers(1, 6))
        shared = rng.permutation(np.arange(1, 200))[:n_shared]
        own = iter(rng.permutation(np.arange(200, 400)))
        tables = np.zeros((B, 10), np.int32)
        lens = []
        for s in range(B):
            L = int(rng.integers(0, 10 * bs + 1))
            tables[s, :n_shared] = shared
            for b in range(n_shared, 10):
                tables[s, b] = next(own)
            lens.append(L)
        assert bench.unique_kv_bytes(tables, lens, 1, 4, bs, 1) == _distinct_slots(tables, lens, bs) * 8


def test_bench_prefix_batch_shares_the_prompt_blocks(pkv):
    """The timed shared-prefix batch: every table starts with the same prompt blocks
    (reference count B), the suffixes are private, and its unique KV bytes are the
    prompt once plus the suffixes."""
    import workloads as wl
    b = wl.make_decode_batch("prefix_beams", with_data=False)
    bs, B = b.block_size, b.num_seqs
    shared = wl.PREFIX_TOKENS // bs
    lens = b.context_lens.astype(np.int64)
    nb = int(np.ceil(1.2 * np.sum(-(-lens // bs))))
    order = wl.rng_for(7).permutation(nb).astype(np.int32)
    mb = int(np.max(-(-lens // bs)))
    bm = bench.build_manager(pkv.BlockManager, nb, bs, order, lens, shared, mb)
    tables, got = bm.export_tables(range(B), mb)
    assert (got == lens).all()
    assert (tables[:, :shared] == tables[0, :shared]).all()
    for blk in tables[0, :shared]:
        assert bm.refcount(int(blk)) == B
    private = [int(x) for s in range(B) for x in tables[s, shared:-(-int(lens[s]) // bs)]]
    assert len(set(private)) == len(private) and not set(private) & set(tables[0, :shared].tolist())
    assert bm.num_free() == nb - shared - len(private)
    per_token = b.num_kv_heads * b.head_dim * 2 * 2
    u = bench.unique_kv_bytes(tables, lens, b.num_kv_heads, b.head_dim, bs)
    assert u == (wl.PREFIX_TOKENS + int((lens - wl.PREFIX_TOKENS).sum())) * per_token
    assert bench.decode_bytes(lens, b.num_heads, b.num_kv_heads, b.head_dim, bs)[0] - u == \
        (B - 1) * wl.PREFIX_TOKENS * per_token
    # every other workload stays unshared
    bm2 = bench.build_manager(pkv.BlockManager, nb, bs, order, lens[:4], 0, mb)
    t2, _ = bm2.export_tables(range(4), mb)
    assert bench.unique_kv_bytes(t2, lens[:4], 8, 128, bs) == bench.decode_bytes(lens[:4], 32, 8, 128, bs)[0]
    bm.close()
    bm2.close()


def test_l2_flush_only_for_small_working_sets():
    import workloads as wl
    per_token = 8 * 128 * 2 * 2
    b = wl.make_decode_batch("prefix_beams", with_data=False)
    lens = b.context_lens.astype(np.int64)
    shared_unique = (wl.PREFIX_TOKENS + int((lens - wl.PREFIX_TOKENS).sum())) * per_token
    assert bench.needs_l2_flush(shared_unique)            # 0.135 GB: flushed
    assert bench.needs_l2_flush(shared_unique // 2)       # the e4m3 pool too
    for name in ("llama7b", "llama13b_mixed_bs16", "long_trace"):
        c = wl.make_decode_batch(name, with_data=False)
        kv = bench.decode_bytes(c.context_lens, c.num_heads, c.num_kv_heads, c.head_dim, c.block_size, 1)[0]
        assert not bench.needs_l2_flush(kv), name         # >= 4x L2 even at one byte per value


def test_beam_ids_group_each_parent_with_its_beams():
    assert bench.beam_ids(3, 1) == [0, 1, 2]
    assert bench.beam_ids(2, 4) == [0, 2, 3, 4, 1, 5, 6, 7]
    ids = bench.beam_ids(128, 4)
    assert sorted(ids) == list(range(512))


def test_bench_beam_batch_matches_the_allocator_model(pkv):
    """The forked shared-prefix batch: the C++ allocator as the bench builds it against
    the reference model driven by the same operations; the first append copies every
    shared partial last block for all beams but the last (which writes in place)."""
    from oracle.block_manager import BlockManagerModel
    import workloads as wl
    bs, parents, beams, shared = 16, 6, 4, 4
    rng = wl.rng_for(11)
    lens = (shared * bs + rng.integers(10, 60, size=parents)).astype(np.int64)
    lens[0] = shared * bs + 32                       # one parent ends on a block boundary: no copy
    nb = 200
    order = rng.permutation(nb).astype(np.int32)
    mb = 16
    bm = bench.build_manager(pkv.BlockManager, nb, bs, order, lens, shared, mb, beams)
    ids = bench.beam_ids(parents, beams)
    model = BlockManagerModel(nb, bs, initial_order=order)
    model.add_seq(0, int(lens[0]))
    prefix = model.tables[0][:shared]
    for s in range(1, parents):
        model.add_seq(s, int(lens[s]), prefix)
    for s in range(parents):
        for k in range(beams - 1):
            model.fork(s, parents + (beams - 1) * s + k)
    for step in range(3):
        slots, pairs = bm.append_slots(ids)
        mslots, mpairs = model.append_slots(ids)
        assert slots.tolist() == list(mslots) and pairs.tolist() == [list(p) for p in mpairs]
        if step == 0:
            partial = int(np.sum(lens % bs != 0))
            assert len(pairs) == (beams - 1) * partial
        else:
            assert len(pairs) == 0
        t, l = bm.export_tables(ids, mb)
        mt, ml = model.export_tables(ids, mb)
        assert t.tolist() == mt and l.tolist() == ml
    for blk in prefix:
        assert bm.refcount(int(blk)) == parents * beams
    # distinct bytes: the prompt once, every parent's full suffix blocks once, each beam's own last block
    u = bench.unique_kv_bytes(t, l, 1, 8, bs, 1)
    assert u == len({int(t[r][p // bs]) * bs + p % bs for r in range(len(ids)) for p in range(int(l[r]))}) * 16
    bm.close()


def test_workload_default_path_is_unforked_and_unshared(pkv):
    """The bench's Workload on the CPU for the tiny batch: ids in order, no beams, no
    shared blocks, the manager's tables and lengths those of plain add_seq calls."""
    import torch
    w = bench.Workload("tiny", 4, seed=3, device=torch.device("cpu"))
    assert list(w.seq_ids) == list(range(w.B)) and w.beams == 1 and w.shared_blocks == 0 and w.layout is None
    assert w.label == "tiny"
    bm = w.new_manager()
    ref = pkv.BlockManager(w.NB, w.bs, w.free_order)
    for s in range(w.B):
        ref.add_seq(s, int(w.lens0[s]) - 1)
    a, b = bm.export_tables(w.seq_ids, w.max_blocks), ref.export_tables(range(w.B), w.max_blocks)
    assert a[0].tolist() == b[0].tolist() and a[1].tolist() == b[1].tolist()
    bm.close()
    ref.close()


def test_every_decode_workload_records_its_length_mix():
    import workloads as wl
    assert set(bench.LENGTH_MIX) == set(wl.WORKLOADS)


def test_pool_usage_shows_what_sharing_saves(pkv):
    import workloads as wl
    b = wl.make_decode_batch("prefix_beams", with_data=False)
    bs, B = b.block_size, b.num_seqs
    lens = b.context_lens.astype(np.int64)
    nb = int(np.ceil(1.2 * np.sum(-(-lens // bs))))
    order = wl.rng_for(7).permutation(nb).astype(np.int32)
    bm = bench.build_manager(pkv.BlockManager, nb, bs, order, lens, wl.PREFIX_TOKENS // bs, int(np.max(-(-lens // bs))))
    u = bench.pool_usage(nb, bm.num_free(), lens, bs)
    ref = int(np.sum(-(-lens // bs)))
    assert u["referenced_by_tables"] == ref and u["used"] == ref - (B - 1) * (wl.PREFIX_TOKENS // bs)
    assert 0.7 < u["saved_by_sharing"] < 0.9 and u["utilisation"] == round(u["used"] / nb, 4)
    plain = bench.pool_usage(nb, nb - ref, lens, bs)
    assert plain["saved_by_sharing"] == 0.0
    bm.close()


def _run_bench(*args):
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    return subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], capture_output=True, text=True,
                          timeout=600, cwd=root)


def test_reference_arm_without_a_device_prints_one_line_and_exits_0():
    import json
    if torch.cuda.is_available():
        import pytest
        pytest.skip("a CUDA device is present; this checks the host-only fallback")
    r = _run_bench("--impl", "reference", "--steps", "2", "--warmup", "3")
    assert r.returncode == 0
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and "unavailable" in out


def test_beams_only_for_the_shared_prefix_workload():
    r = _run_bench("--workload", "llama7b", "--beams", "4", "--warmup", "3")
    assert r.returncode != 0 and "prefix_beams only" in r.stderr


class _FakeEvent:
    def __init__(self, enable_timing=False):
        self.recorded = False

    def record(self, stream=None):
        self.recorded = True

    def synchronize(self):
        assert self.recorded, "waited on an event that was never recorded"

    def elapsed_time(self, other):
        return 2.0


class _FakeStream:
    def __init__(self, device=None):
        pass

    def wait_event(self, ev):
        pass

    def synchronize(self):
        pass


def test_e2e_host_logic_with_stand_in_streams(pkv, monkeypatch):
    """The e2e harness's host logic on the CPU: streams, events and pinning replaced by
    stand-ins and the three kernels by stubs (the stub decode writes a known output).
    Checks the per-step byte accounting, the KV bytes and that every step's output is
    read back once."""
    import contextlib
    import types
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: _FakeStream())
    monkeypatch.setattr(torch.cuda, "Stream", _FakeStream)
    monkeypatch.setattr(torch.cuda, "Event", _FakeEvent)
    monkeypatch.setattr(torch.cuda, "stream", lambda s: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    w = bench.Workload("tiny", 8, seed=5, device=torch.device("cpu"))
    calls = {"write": 0, "decode": 0, "copy": 0}

    def write(k, v, slots, status):
        assert k.shape == (w.B, w.Hkv, w.D) and slots.shape == (w.B,)
        calls["write"] += 1

    def decode(out, q, tables, lens, max_len, ws, path, status, shared=None):
        assert q.shape == (w.B, w.Hq, w.D) and tables.shape == (w.B, w.max_blocks) and lens.shape == (w.B,)
        out.fill_(1.0)
        calls["decode"] += 1

    w.write, w.decode = write, decode
    w.copy = lambda pairs, status: calls.__setitem__("copy", calls["copy"] + 1)
    args = types.SimpleNamespace(steps=4, e2e_steps=4, warmup=3)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16)
    res = bench.run_e2e(args, w, pkv, torch.device("cpu"), 0, None, out, None, 1024)
    assert calls["write"] == calls["decode"] == 7 and calls["copy"] == 0
    per_step_in = 2 * w.B * (w.Hq + 2 * w.Hkv) * w.D + 8 * w.B + 4 * w.B * w.max_blocks + 4 * w.B
    assert res["h2d_bytes_per_step"] == per_step_in
    assert res["d2h_bytes_per_step"] == 2 * w.B * w.Hq * w.D
    assert res["steps"] == 4 and res["ms_per_step"] == 0.5
    # KV of the timed steps: the allocator's lengths at steps 3..6 (lens0 at step 0)
    kv = sum(int((w.lens0 + i).sum()) for i in range(3, 7)) * w.Hkv * w.D * 2 * 2
    assert res["value"] == round(kv / (2.0 * 1e-3) / 1e9, 1)


class _FakeClocks:
    def __init__(self, device):
        pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False

    def summary(self):
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": []}


def _stand_in_run_ours(monkeypatch, pkv, calls, **overrides):
    import contextlib
    import types
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: _FakeStream())
    monkeypatch.setattr(torch.cuda, "Stream", _FakeStream)
    monkeypatch.setattr(torch.cuda, "Event", _FakeEvent)
    monkeypatch.setattr(torch.cuda, "stream", lambda s: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a, **k: None)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    monkeypatch.setattr(bench, "bench_device", lambda local_rank: torch.device("cpu"))
    monkeypatch.setattr(bench, "ClockSampler", _FakeClocks)
    monkeypatch.setattr(bench, "stream_read_gbs", lambda pkv, device: 7000.0)

    def count(name):
        def f(self, *a, **k):
            calls[name] = calls.get(name, 0) + 1
        return f
    monkeypatch.setattr(bench.Workload, "write", count("write"))
    monkeypatch.setattr(bench.Workload, "copy", count("copy"))
    monkeypatch.setattr(bench.Workload, "decode", count("decode"))
    args = types.SimpleNamespace(workload="tiny", steps=5, warmup=3, states=4, e2e_steps=3, kv="bf16", path="auto",
                                 beams=1, no_e2e=False, no_cpu_baseline=True, cpu_budget=1.0)
    for k, v in overrides.items():
        setattr(args, k, v)
    return bench.run_ours(args, 0, 1, 0)


def test_run_ours_host_logic_with_stand_ins(pkv, monkeypatch):
    """The decode bench's host logic on the CPU (stand-in streams, events, clocks and
    kernels) for the tiny batch: every contract key, the launch count, the L2 flush of a
    small working set, and distinct bytes equal to logical bytes with nothing shared."""
    calls = {}
    res = _stand_in_run_ours(monkeypatch, pkv, calls)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in res, key
    assert calls["decode"] == 3 + 5 + 3 + 3 and "copy" not in calls   # warm-up, timed, e2e warm-up and timed
    assert res["gpu_launches"] == 5 * 3                                # write, plan, decode per step (no split)
    assert res["config"]["l2"].startswith("L2 flushed")                # 29 KB of KV is far below 4x L2
    assert res["config"]["pool"]["saved_by_sharing"] == 0.0
    r = res["roofline"]
    assert r["algorithmic_bytes_per_launch"] == r["logical_bytes_per_launch"]
    assert res["ms_per_step"] == 2.0                                   # the stand-in events' elapsed time
    import json
    json.dumps(res)                                                    # the line main() prints


def test_run_ours_beam_phase_with_stand_ins(pkv, monkeypatch):
    """The shared-prefix batch forked into 4 beams (6 prompts here): copies on the first
    prepared step only, distinct bytes well below logical, sharing visible in the pool."""
    import workloads as wl
    orig = wl.make_decode_batch
    monkeypatch.setattr(wl, "make_decode_batch", lambda name, **k: orig(name, num_seqs=6, **k))
    calls = {}
    res = _stand_in_run_ours(monkeypatch, pkv, calls, workload="prefix_beams", beams=4, steps=4, states=4)
    cfg = res["config"]
    assert cfg["num_seqs"] == 24 and cfg["beams"] == 4 and cfg["workload"] == "prefix_beams+beams4"
    assert cfg["pool"]["saved_by_sharing"] > 0.5
    r = res["roofline"]
    assert r["algorithmic_bytes_per_launch"] < 0.5 * r["logical_bytes_per_launch"]
    assert r["traffic"] is None                      # the capture was of the 128-prompt batch
    # the first prepared step carries the copies; timed steps replay states 3, 0, 1, 2
    assert calls.get("copy", 0) >= 1
    import json
    json.dumps(res)


def test_run_ours_shared_prefix_over_an_8bit_pool_with_stand_ins(pkv, monkeypatch):
    """The shared-prompt batch over an 8-bit pool takes the shared-prefix decode: launches per
    step include the widening of the shared blocks and the query split."""
    import workloads as wl
    orig = wl.make_decode_batch
    monkeypatch.setattr(wl, "make_decode_batch", lambda name, **k: orig(name, num_seqs=6, **k))
    calls = {}
    res = _stand_in_run_ours(monkeypatch, pkv, calls, workload="prefix_beams", kv="fp8", steps=4, states=4)
    cfg = res["config"]
    assert cfg["decode"] == "shared-prefix" and cfg["kv_dtype"] == "fp8"
    r = res["roofline"]
    assert r["kernel"].startswith("paged_attention_decode_shared_fp8")
    assert r["algorithmic_bytes_per_launch"] < r["logical_bytes_per_launch"]
    # per step: write, setup, widening + shared phase, plan, query split, decode, merge
    assert res["gpu_launches"] == 4 * 8
    import json
    json.dumps(res)


def test_recorded_traffic_only_for_the_captured_batch(tmp_path, monkeypatch):
    """A recorded ncu figure is reported only for the kernel sources, table layout and batch
    size it was captured on."""
    import json
    (tmp_path / "profiles").mkdir()
    digest = bench.source_digest("decode_simt")
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({
        "b": {"dram_bytes_per_launch": 1234, "sources": digest, "algorithmic_per_launch": 1000},
        "shared": {"dram_bytes_per_launch": 99, "sources": digest, "algorithmic_per_launch": 10, "layout": "x"}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_digest", lambda kind: digest)
    assert bench.recorded_traffic("b", "decode_simt", 1000) == 1234
    assert bench.recorded_traffic("b", "decode_simt", 1040) == round(1234 * 1.04)  # more steps: scaled
    assert bench.recorded_traffic("b", "decode_simt", 900) is None          # another batch size
    assert bench.recorded_traffic("b", "decode_simt", 1000, "x") is None    # another layout
    assert bench.recorded_traffic("shared", "decode_simt", 10, "x") == 99
    assert bench.recorded_traffic("missing", "decode_simt", 1000) is None
    monkeypatch.setattr(bench, "source_digest", lambda kind: "changed")
    assert bench.recorded_traffic("b", "decode_simt", 1000) is None          # sources changed


@pytest.mark.parametrize("oracle_leg", [False, True])
def test_run_trace_host_logic_with_stand_ins(pkv, monkeypatch, oracle_leg):
    """The continuous-batching trace bench on the CPU with a shrunken trace (4 slots,
    short contexts, small pool) and stubbed kernels: admissions, frees and the recorded
    readings, allocator time reported, seq-steps with it below those without; with the
    oracle leg, one sampled sequence per 20 timed steps is stashed and checked after the loop."""
    import contextlib
    import types
    import workloads as wl
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: _FakeStream())
    monkeypatch.setattr(torch.cuda, "Event", _FakeEvent)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a, **k: None)
    monkeypatch.setattr(bench, "bench_device", lambda local_rank: torch.device("cpu"))
    monkeypatch.setattr(bench, "ClockSampler", _FakeClocks)
    orig = wl.TraceParams
    monkeypatch.setattr(wl, "TraceParams", lambda steps: orig(max_batch=4, num_heads=8, num_kv_heads=2, head_dim=64,
                                                             block_size=16, len_lo=40, len_hi=120, budget_lo=1,
                                                             budget_hi=6, steps=steps, num_blocks=256))
    kernel_calls = {"decode": 0, "write": 0}
    monkeypatch.setattr(pkv, "reshape_and_cache",
                        lambda *a, **k: kernel_calls.__setitem__("write", kernel_calls["write"] + 1))
    monkeypatch.setattr(pkv, "paged_attention_decode",
                        lambda *a, **k: kernel_calls.__setitem__("decode", kernel_calls["decode"] + 1))
    monkeypatch.setattr(pkv, "copy_blocks", lambda *a, **k: None)
    args = types.SimpleNamespace(steps=20, warmup=3, no_cpu_baseline=not oracle_leg)
    res = bench.run_trace(args, 0, 1, 0)
    if oracle_leg:
        cb = res["cpu_baseline"]
        assert cb["kind"] == "oracle" and cb["cores"] == 1 and "1 sequences" in cb["sample"], cb
    else:
        assert "cpu_baseline" not in res
    cfg = res["config"]
    assert cfg["workload"] == "long_trace_continuous" and cfg["admitted"] > 4
    assert cfg["initial_lengths"] == "U{40..120}" and cfg["budgets"] == "U{1..6}"
    assert cfg["arrivals"].startswith("Bernoulli(0.5) per free slot per step")
    assert 0 < kernel_calls["decode"] <= 23
    assert res["allocator_us_per_step"] > 0
    assert res["seq_steps_per_s_with_allocator"] < res["seq_steps_per_s"]
    assert res["ms_per_step_span"] > 0   # first kernel start to last kernel end, launch gaps included
    import json
    json.dumps(res)


def test_cpu_baseline_leg_with_stand_ins(pkv, monkeypatch):
    """The oracle leg of the decode line (1 core, then every core over spawned workers)
    on the tiny batch, through the same stand-ins."""
    calls = {}
    res = _stand_in_run_ours(monkeypatch, pkv, calls, no_cpu_baseline=False, cpu_budget=1.0)
    cb = res["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] > 0 and cb["unit"] == "GB/s"
    assert "tiny batch" in cb["sample"]
    assert cb["all_cores"]["cores"] >= 1 and cb["all_cores"]["value"] > 0


def test_run_prefill_host_logic_with_stand_ins(pkv, monkeypatch):
    """The chunked-prefill line on the CPU with a shrunken batch and stubbed kernels:
    contract keys, launches, FLOPs per step, and the e2e byte counts."""
    import contextlib
    import json
    import types
    import workloads as wl
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: _FakeStream())
    monkeypatch.setattr(torch.cuda, "Event", _FakeEvent)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a, **k: None)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    monkeypatch.setattr(bench, "bench_device", lambda local_rank: torch.device("cpu"))
    monkeypatch.setattr(bench, "ClockSampler", _FakeClocks)
    orig = wl.make_prefill_batch
    monkeypatch.setattr(wl, "make_prefill_batch",
                        lambda name, **k: orig(name, num_seqs=3, length_scale=0.05, num_heads=8, num_kv_heads=4, **k))
    calls = {"write": 0, "prefill": 0}
    monkeypatch.setattr(pkv, "reshape_and_cache", lambda *a, **k: calls.__setitem__("write", calls["write"] + 1))
    monkeypatch.setattr(pkv, "paged_attention_prefill",
                        lambda *a, **k: calls.__setitem__("prefill", calls["prefill"] + 1))
    args = types.SimpleNamespace(workload="chunked_prefill_13b", steps=4, warmup=3, e2e_steps=2,
                                 no_cpu_baseline=True, cpu_budget=1.0)
    res = bench.run_prefill(args, 0, 1, 0)
    json.dumps(res)
    assert calls["prefill"] == 3 + 4 + 2 and calls["write"] == calls["prefill"]
    cfg = res["config"]
    T, Hq, Hkv, D = cfg["query_tokens"], cfg["num_heads"], cfg["num_kv_heads"], cfg["head_dim"]
    assert (Hq, Hkv) == (8, 4) and T == sum(cfg["query_lens"])
    assert cfg["flops_per_step"] == bench.prefill_flops(np.array(cfg["query_lens"]), np.array(cfg["context_lens"]),
                                                        Hq, D)
    assert res["gpu_launches"] == 3 * 4 and res["roofline"]["bound"] == "tensor"
    assert res["e2e"]["h2d_bytes_per_step"] == 2 * T * (Hq + 2 * Hkv) * D
    assert res["e2e"]["d2h_bytes_per_step"] == 2 * T * Hq * D


def test_run_swap_host_logic_with_stand_ins(pkv, monkeypatch):
    """The swap line on the CPU with small blocks and a stubbed swap kernel: four calls
    per step (K and V out, K and V in), bytes per step, and the JSON line."""
    import json
    import types
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: _FakeStream())
    monkeypatch.setattr(torch.cuda, "Event", _FakeEvent)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a, **k: None)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    monkeypatch.setattr(bench, "bench_device", lambda local_rank: torch.device("cpu"))
    monkeypatch.setattr(bench, "ClockSampler", _FakeClocks)
    monkeypatch.setattr(bench, "SWAP_SHAPE", (2, 16, 8))
    seen = []
    monkeypatch.setattr(pkv, "swap_blocks", lambda src, dst, pairs, **k: seen.append((src.shape[0], dst.shape[0],
                                                                                        tuple(pairs.shape))))
    args = types.SimpleNamespace(steps=5, warmup=3, no_cpu_baseline=True, cpu_budget=1.0)
    res = bench.run_swap(args, 0, 1, 0)
    json.dumps(res)
    assert len(seen) == 4 * (3 + 5)
    assert {s[2] for s in seen} == {(bench.SWAP_PAIRS, 2)}
    assert seen[0][:2] == (4096, 1024) and seen[2][:2] == (1024, 4096)      # out to the host pool, then back in
    block = 2 * 16 * 8 * 2
    assert res["config"]["block_bytes"] == block and res["config"]["bytes_per_step"] == 4 * bench.SWAP_PAIRS * block


def test_reference_arm_with_stand_ins(monkeypatch):
    """The reference arm (the oracle timed on the host) on the tiny batch, its device
    stood in by the CPU: the JSON line with impl, cpu_baseline and a zero-copy e2e.
    The library is made unimportable for the call: the arm depends on nothing it ships."""
    import json
    import sys
    import types
    monkeypatch.setitem(sys.modules, "paged_kv_cache_423_b200", None)
    monkeypatch.setattr(torch.cuda, "is_available", lambda: True)
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a, **k: None)
    monkeypatch.setattr(bench, "bench_device", lambda local_rank: torch.device("cpu"))
    args = types.SimpleNamespace(workload="tiny", steps=2, warmup=3, kv="bf16", beams=1, ref_budget=2.0,
                                 cpu_budget=1.0)
    res = bench.run_reference(args, 0, 1, 0)
    json.dumps(res)
    assert res["impl"] == "reference" and res["value"] > 0 and res["unit"] == "GB/s"
    assert res["cpu_baseline"]["kind"] == "oracle" and res["cpu_baseline"]["value"] == res["value"]
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["e2e"]["d2h_bytes_per_step"] == 0
    assert res["config"]["workload"] == "tiny"


@pytest.mark.parametrize("workload,beams", [("prefix_beams", 1), ("prefix_beams", 4), ("llama7b", 1)])
def test_reference_arm_tables_equal_the_native_ones(pkv, workload, beams):
    """The reference arm builds its batch with the allocator's reference model; the same
    operations on the C++ allocator give the same tables, lengths, slots and copy pairs."""
    w = bench.Workload(workload, 2, seed=1000, device=torch.device("cpu"), beams=beams, native=False)
    assert w.pkv is None
    native = bench.build_manager(pkv.BlockManager, w.NB, w.bs, w.free_order, w.parent_lens0 - 1, w.shared_blocks,
                                 w.max_blocks, w.beams)
    model = w.new_manager()
    for _ in range(2):
        a, b = native.append_slots(w.seq_ids), model.append_slots(w.seq_ids)
        assert a[0].tolist() == b[0].tolist() and a[1].tolist() == b[1].tolist()
        ta, la = native.export_tables(w.seq_ids, w.max_blocks)
        tb, lb = model.export_tables(w.seq_ids, w.max_blocks)
        assert ta.dtype == tb.dtype and ta.tolist() == tb.tolist() and la.tolist() == lb.tolist()
    assert native.num_free() == model.num_free()
    native.close()


def test_reference_prefill_batch_without_the_library(pkv, monkeypatch):
    """The prefill reference leg's batch from the allocator's reference model equals the
    native one (slots, tables, lengths), with the library unimportable while it is built."""
    import sys
    native = bench.PrefillWorkload("chunked_prefill_13b", 1, seed=2000, device=torch.device("cpu"))
    monkeypatch.setitem(sys.modules, "paged_kv_cache_423_b200", None)
    ref = bench.PrefillWorkload("chunked_prefill_13b", 1, seed=2000, device=torch.device("cpu"), native=False)
    assert ref.pkv is None and ref.ws is None
    for k in ("slots", "tables", "lens", "qstart"):
        assert torch.equal(getattr(native, k), getattr(ref, k)), k


def test_shared_decode_applies_only_where_it_can_run():
    import types
    args = lambda shared="auto", path="auto": types.SimpleNamespace(shared=shared, path=path)  # noqa: E731
    w = lambda kv8=False, shared_blocks=64, Hq=32, Hkv=8, D=128: types.SimpleNamespace(  # noqa: E731
        kv8=kv8, shared_blocks=shared_blocks, Hq=Hq, Hkv=Hkv, D=D)
    assert bench.shared_decode_applies(args(), w())                    # the shared-prompt batch
    assert not bench.shared_decode_applies(args(), w(shared_blocks=0))  # nothing shared: plain decode
    assert bench.shared_decode_applies(args("on"), w(shared_blocks=0))
    assert not bench.shared_decode_applies(args("off"), w())
    assert bench.shared_decode_applies(args(), w(kv8=True))            # the 8-bit pool too
    assert not bench.shared_decode_applies(args(path="simt"), w())
    assert not bench.shared_decode_applies(args(), w(Hq=40, Hkv=40))   # MHA: no tensor-core decode
    with pytest.raises(SystemExit):
        bench.shared_decode_applies(args("on"), w(Hq=40, Hkv=40))


def test_e2e_shared_prefix_plan_travels_with_each_step(pkv, monkeypatch):
    """With the shared-prefix decode the e2e harness plans every step on the host, straight
    into the pinned buffer, and the plan's bytes count as host-to-device traffic; the decode
    gets the device plan, its info and the shared workspace."""
    import contextlib
    import types
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: _FakeStream())
    monkeypatch.setattr(torch.cuda, "Stream", _FakeStream)
    monkeypatch.setattr(torch.cuda, "Event", _FakeEvent)
    monkeypatch.setattr(torch.cuda, "stream", lambda s: contextlib.nullcontext())
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    w = bench.Workload("tiny", 8, seed=5, device=torch.device("cpu"))
    sws = torch.empty(16, dtype=torch.uint8)
    seen = []

    def decode(out, q, tables, lens, max_len, ws, path, status, shared=None):
        plan, info, ws_shared = shared
        assert ws_shared is sws and plan.dtype == torch.uint8 and plan.numel() >= info.bytes
        seen.append(int(info.bytes))
        out.fill_(1.0)

    w.write, w.decode = (lambda *a, **k: None), decode
    w.copy = lambda pairs, status: None
    args = types.SimpleNamespace(steps=4, e2e_steps=4, warmup=3)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16)
    res = bench.run_e2e(args, w, pkv, torch.device("cpu"), 0, None, out, None, 1024, sws)
    assert len(seen) == 7 and all(b > 0 for b in seen)
    plain = 2 * w.B * (w.Hq + 2 * w.Hkv) * w.D + 8 * w.B + 4 * w.B * w.max_blocks + 4 * w.B
    assert res["h2d_bytes_per_step"] == plain + sum(seen[3:]) // 4


def test_shared_private_rule_matches_the_library():
    """bench.py counts the 8-bit query split only when the shared-prefix decode's private phase
    is on the tensor cores; its remainder bound must be the library's."""
    import re
    src = open(os.path.join(bench.ROOT, "paged_kv_cache_423_b200", "csrc", "shared_decode.cu")).read()
    m = re.search(r"#define PKV_SHARED_SIMT_MAX (\d+)", src)
    assert m and int(m.group(1)) == bench.SHARED_SIMT_SUFFIX_MAX


def test_shared_plan_options_by_pool():
    """Segments of 2 rows over bf16 pools and of 5 over 8-bit pools unless --min-rows says
    otherwise."""
    import types
    assert bench.shared_min_rows(types.SimpleNamespace(kv="bf16")) == 2
    assert bench.shared_min_rows(types.SimpleNamespace(kv="fp8")) == 5
    assert bench.shared_min_rows(types.SimpleNamespace(kv="fp8", min_rows=3)) == 3
    assert bench.shared_min_rows(types.SimpleNamespace(kv="bf16", min_rows=None)) == 2
