"""The C-ABI library on the host: it loads, exports every declared symbol, rejects
bad arguments before touching a GPU, and its block manager matches the reference
model of the allocator operation for operation (all CPU-only)."""
import ctypes
import os
import re

import numpy as np
import pytest

import workloads as wl
from oracle.block_manager import BlockManagerError, BlockManagerModel

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"PKV_API\s+[\w\s\*]*?\b(pkv_\w+)\s*\(", text))
    return sorted(names)


def test_library_loads_and_exports_every_declared_symbol(pkv):
    lib = pkv.library()
    names = declared_symbols()
    assert len(names) >= 20
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert lib.pkv_version() >= 10000


def test_binding_covers_every_symbol(pkv):
    from paged_kv_cache_423_b200 import _SIGNATURES
    assert set(declared_symbols()) <= set(_SIGNATURES)


def test_header_entry_points_cite_their_passage():
    text = open(os.path.join(ROOT, "include", "pkv.h")).read()
    for anchor in ("§2.1", "§1.4", "内存共享", "LLM serving的基本流程与KV缓存", "vLLM的核心创新"):
        assert anchor in text


def test_argument_errors_before_any_device_work(pkv):
    lib = pkv.library()
    fake = ctypes.c_void_p(0x1000)
    # unsupported head_dim / block size / grouping; bad out dtype; misaligned pointer
    args = dict(out=fake, out_dtype=0, query=fake, kc=fake, vc=fake, tables=fake, max_blocks=4, lens=fake,
                max_ctx=64, B=2, Hq=4, Hkv=2, D=128, bs=16, NB=8, scale=0.1, part=0, path=0, ws=fake,
                ws_bytes=1 << 20)

    def call(**kw):
        a = dict(args, **kw)
        return lib.pkv_paged_attention_decode(a["out"], a["out_dtype"], a["query"], a["kc"], a["vc"], a["tables"],
                                              a["max_blocks"], a["lens"], a["max_ctx"], a["B"], a["Hq"], a["Hkv"],
                                              a["D"], a["bs"], a["NB"], a["scale"], a["part"], a["path"], a["ws"],
                                              a["ws_bytes"], None, None)

    assert call(D=96) == pkv.PKV_ERR_UNSUPPORTED
    assert call(bs=8) == pkv.PKV_ERR_UNSUPPORTED
    assert call(Hq=5) == pkv.PKV_ERR_UNSUPPORTED
    assert call(Hq=70000, Hkv=70000) == pkv.PKV_ERR_UNSUPPORTED  # kv head ids are 16-bit in the kernels
    assert call(out_dtype=7) == pkv.PKV_ERR_INVALID
    assert call(part=100) == pkv.PKV_ERR_INVALID
    assert call(query=ctypes.c_void_p(0x1008)) == pkv.PKV_ERR_INVALID
    assert call(ws=ctypes.c_void_p(0x1010)) == pkv.PKV_ERR_INVALID
    assert call(ws_bytes=16) == pkv.PKV_ERR_INVALID
    assert b"workspace" in lib.pkv_last_error_string()
    assert call(B=0) == pkv.PKV_OK       # empty batch: nothing to do
    assert lib.pkv_reshape_and_cache(fake, fake, fake, fake, fake, 4, 8, 2, 96, 16, None, None) == pkv.PKV_ERR_UNSUPPORTED
    assert lib.pkv_reshape_and_cache(fake, fake, fake, fake, fake, 0, 8, 2, 128, 16, None, None) == pkv.PKV_OK
    assert lib.pkv_copy_blocks(None, None, 0, None, 0, 8, 4096, None, None) == pkv.PKV_OK
    assert lib.pkv_copy_blocks(None, None, 1, None, 3, 8, 4095, None, None) == pkv.PKV_ERR_INVALID
    # the bandwidth reference: sizes and alignment are checked before any launch
    assert lib.pkv_stream_read(fake, 0, fake, None) == pkv.PKV_OK
    assert lib.pkv_stream_read(fake, 40, fake, None) == pkv.PKV_ERR_INVALID
    assert lib.pkv_stream_read(None, 64, fake, None) == pkv.PKV_ERR_INVALID
    assert lib.pkv_stream_read(ctypes.c_void_p(0x1008), 64, fake, None) == pkv.PKV_ERR_INVALID
    assert lib.pkv_stream_read(fake, 64, ctypes.c_void_p(0x1002), None) == pkv.PKV_ERR_INVALID


def test_prefill_argument_errors_before_any_device_work(pkv):
    lib = pkv.library()
    fake = ctypes.c_void_p(0x1000)
    args = dict(out=fake, out_dtype=0, query=fake, kc=fake, vc=fake, tables=fake, max_blocks=4, qstart=fake,
                lens=fake, B=2, T=10, max_ctx=64, Hq=8, Hkv=2, D=128, bs=16, NB=8, scale=0.1, ws=fake,
                ws_bytes=1 << 20)

    def call(**kw):
        a = dict(args, **kw)
        return lib.pkv_paged_attention_prefill(a["out"], a["out_dtype"], a["query"], a["kc"], a["vc"], a["tables"],
                                               a["max_blocks"], a["qstart"], a["lens"], a["B"], a["T"],
                                               a["max_ctx"], a["Hq"], a["Hkv"], a["D"], a["bs"], a["NB"],
                                               a["scale"], a["ws"], a["ws_bytes"], None, None)
    assert call(D=64) == pkv.PKV_ERR_UNSUPPORTED          # the tensor-core prefill is head_dim 128
    assert call(bs=8) == pkv.PKV_ERR_UNSUPPORTED
    assert call(Hq=6, Hkv=2) == pkv.PKV_ERR_UNSUPPORTED   # group 3 does not divide 128
    assert call(Hq=7) == pkv.PKV_ERR_UNSUPPORTED
    assert call(out_dtype=3) == pkv.PKV_ERR_INVALID
    assert call(T=-1) == pkv.PKV_ERR_INVALID
    assert call(query=ctypes.c_void_p(0x1004)) == pkv.PKV_ERR_INVALID
    assert call(ws=ctypes.c_void_p(0x1080)) == pkv.PKV_ERR_INVALID
    assert call(ws_bytes=64) == pkv.PKV_ERR_INVALID
    assert b"workspace" in lib.pkv_last_error_string()
    assert call(qstart=None) == pkv.PKV_ERR_INVALID
    for bad_scale in (0.0, -0.1, float("inf"), float("nan")):  # hidden keys are -inf scores
        assert call(scale=bad_scale) == pkv.PKV_ERR_INVALID
        assert b"scale" in lib.pkv_last_error_string()
    assert call(T=0) == pkv.PKV_OK                        # no rows: nothing to do
    assert call(B=0) == pkv.PKV_OK


def test_prefill_workspace_size(pkv):
    # 256 bytes of counters + one 16-byte entry per pair of 128-row query tiles (upper
    # bound: T / (2 * 128 / g) + B), rounded up to 256 bytes
    def up(x):
        return -(-x // 256) * 256
    assert pkv.paged_attention_prefill_workspace_size(8, 4096, 40, 40) == 256 + up(16 * (16 + 8))
    assert pkv.paged_attention_prefill_workspace_size(8, 4096, 64, 8) == 256 + up(16 * (128 + 8))
    assert pkv.paged_attention_prefill_workspace_size(1, 1, 128, 1) == 256 + up(16 * 2)
    with pytest.raises(pkv.PkvError):
        pkv.paged_attention_prefill_workspace_size(2, 10, 6, 2)


def test_workspace_size_and_partition_choice(pkv):
    assert pkv.paged_attention_partition_tokens(256, 40, 16, 2000) == 512
    assert pkv.paged_attention_partition_tokens(4, 2, 16, 33) == 64
    small = pkv.paged_attention_workspace_size(4, 2, 2, 64, 16, 33)
    big = pkv.paged_attention_workspace_size(16, 64, 8, 128, 32, 32000)
    assert 0 < small < big
    # partials: B * Hq * parts * (D + 2) floats dominate
    assert big >= 16 * 64 * 63 * 130 * 4
    with pytest.raises(pkv.PkvError):
        pkv.paged_attention_workspace_size(4, 2, 2, 64, 16, 33, partition_tokens=48)


# ---------------------------------------------------------------------------
# Block manager: C++ vs the reference model, operation by operation
# ---------------------------------------------------------------------------

def same_state(cpp, model: BlockManagerModel):
    assert cpp.num_free() == model.num_free()
    assert cpp.free_list() == list(model.free)
    for b in range(model.num_blocks):
        assert cpp.refcount(b) == model.ref[b]
    assert cpp.num_host_free() == model.num_host_free()
    for b in range(len(model.host_ref)):
        assert cpp.host_refcount(b) == model.host_ref[b]
    assert cpp.num_cached_blocks() == model.num_cached_blocks()
    for s in model.tables:
        assert cpp.is_swapped(s) == model.is_swapped(s)
    ids = sorted(s for s in model.tables if not model.is_swapped(s))
    if ids:
        mb = max(len(t) for t in model.tables.values()) or 1
        tables, lens = cpp.export_tables(ids, mb)
        exp_t, exp_l = model.export_tables(ids, mb)
        assert tables.tolist() == exp_t and lens.tolist() == exp_l


def run_both(op, cpp, model, pkv):
    """Run op on both; they must agree on success or on the error code."""
    err_m = err_c = None
    res_m = res_c = None
    try:
        res_m = op(model)
    except BlockManagerError as e:
        err_m = e.code
    try:
        res_c = op(cpp)
    except pkv.PkvError as e:
        err_c = e.code
    assert err_m == err_c
    return res_m, res_c


@pytest.mark.parametrize("seed", range(5))
@pytest.mark.parametrize("extended", [False, True], ids=["base", "swap_and_prefix_cache"])
def test_block_manager_matches_model(pkv, seed, extended):
    rng = wl.rng_for(100 + seed)
    nb, bs = 40, 4
    order = rng.permutation(nb).astype(np.int32)
    hb = 20 if extended else 0
    cpp = pkv.BlockManager(nb, bs, order, num_host_blocks=hb)
    model = BlockManagerModel(nb, bs, order, num_host_blocks=hb)
    prompts = [list(rng.integers(0, 4, size=30)) for _ in range(3)]
    texts = {}  # seq -> token ids when known (prompt-token sequences and their decode appends)
    next_id = 0
    for _ in range(300):
        every = sorted(model.tables)
        live = [x for x in every if not model.is_swapped(x)]
        gone = [x for x in every if model.is_swapped(x)]
        op = int(rng.integers(0, 11 if extended else 6))
        if op == 9 and live:
            # decode appends with token ids: blocks they complete register in the prefix cache
            pick = [int(x) for x in rng.permutation(live)[:int(rng.integers(1, len(live) + 1))]]
            toks = [int(t) for t in rng.integers(0, 4, size=len(pick))]
            (sm, pm), (sc, pc) = [r if r is not None else (None, None) for r in run_both(
                lambda m: m.append_tokens(pick, toks), cpp, model, pkv)]
            if sm is not None:
                assert list(sc) == sm and [tuple(p) for p in pc.tolist()] == pm
                for s_, t_ in zip(pick, toks):
                    if texts.get(s_) is not None:
                        texts[s_] = texts[s_] + [t_]
            same_state(cpp, model)
            continue
        if op == 10:
            # a prompt continuing a generated text
            known = [x for x in live if texts.get(x) is not None]
            if known:
                src = known[int(rng.integers(len(known)))]
                toks = texts[src] + [int(t) for t in rng.integers(0, 4, size=int(rng.integers(1, 3)))]
                sid = next_id
                next_id += 1
                rm, rc = run_both(lambda m: m.add_seq_tokens(sid, toks), cpp, model, pkv)
                assert rm == rc
                if rm is not None:
                    texts[sid] = toks
            same_state(cpp, model)
            continue
        if op >= 6 and op <= 8:
            # swap out / swap in (sometimes of a sequence in the wrong pool) / prompt admission
            if op == 6 and every:
                pick = [int(x) for x in rng.permutation(every)[:int(rng.integers(1, min(3, len(every)) + 1))]]
                rm, rc = run_both(lambda m: m.swap_out(pick), cpp, model, pkv)
                if rm is not None:
                    assert [tuple(p) for p in rc.tolist()] == rm
            elif op == 7 and every:
                pick = [int(x) for x in rng.permutation(gone if gone and rng.random() < 0.8 else every)
                        [:int(rng.integers(1, 3))]]
                rm, rc = run_both(lambda m: m.swap_in(pick), cpp, model, pkv)
                if rm is not None:
                    assert [tuple(p) for p in rc.tolist()] == rm
            else:
                p = prompts[int(rng.integers(len(prompts)))]
                toks = p[:int(rng.integers(1, len(p) + 1))] + [int(t) for t in rng.integers(0, 4, size=int(rng.integers(0, 3)))]
                sid = next_id
                next_id += 1
                rm, rc = run_both(lambda m: m.add_seq_tokens(sid, toks), cpp, model, pkv)
                assert rm == rc
                if rm is not None:
                    texts[sid] = [int(t) for t in toks]
            same_state(cpp, model)
            continue
        if not live:
            op = 0
        if op == 0:
            shared = []
            if live and rng.random() < 0.5:
                donor = live[int(rng.integers(len(live)))]
                shared = model.tables[donor][:int(rng.integers(0, model.lens[donor] // bs + 1))]
            n_tok = len(shared) * bs + int(rng.integers(0, 10))
            sid = next_id
            next_id += 1
            run_both(lambda m: m.add_seq(sid, n_tok, shared), cpp, model, pkv)
        elif op == 1:
            parent = live[int(rng.integers(len(live)))]
            child = next_id
            next_id += 1
            run_both(lambda m: m.fork(parent, child), cpp, model, pkv)
            texts[child] = None if texts.get(parent) is None else list(texts[parent])
        elif op == 2:
            pick = [int(s) for s in rng.permutation(live)[:int(rng.integers(1, len(live) + 1))]]
            (sm, pm), (sc, pc) = [r if r is not None else (None, None) for r in run_both(
                lambda m: m.append_slots(pick), cpp, model, pkv)]
            if sm is not None:
                assert list(sc) == sm and [tuple(p) for p in pc.tolist()] == pm
                for s_ in pick:
                    texts[s_] = None
        elif op == 3:
            victim = every[int(rng.integers(len(every)))]
            run_both(lambda m: m.free_seq(victim), cpp, model, pkv)
        elif op == 4:
            s = live[int(rng.integers(len(live)))]
            L = model.lens[s]
            rm, rc = run_both(lambda m: m.slots(s, 0, L), cpp, model, pkv)
            assert list(rc) == rm
        else:
            bad = int(rng.integers(-2, nb + 2))
            run_both(lambda m: m.decref(bad) if m.refcount(bad) == 0 else m.incref(bad), cpp, model, pkv)
        same_state(cpp, model)
    cpp.close()


def test_block_manager_errors_and_oom(pkv):
    bm = pkv.BlockManager(3, 4, [2, 0, 1])
    bm.add_seq(0, 4)
    bm.add_seq(1, 4)
    with pytest.raises(pkv.PkvError) as e:
        bm.append_slots([0, 1])
    assert e.value.code == pkv.PKV_ERR_OOM
    assert bm.num_free() == 1 and bm.seq_len(0) == 4 and bm.seq_len(1) == 4
    with pytest.raises(pkv.PkvError) as e:
        bm.append_slots([0, 0])
    assert e.value.code == pkv.PKV_ERR_INVALID
    with pytest.raises(pkv.PkvError):
        pkv.BlockManager(4, 4, [0, 1, 1, 2])


def test_block_manager_cow_example(pkv):
    bm = pkv.BlockManager(16, 4)
    bm.add_seq(0, 6)
    for c in (1, 2, 3):
        bm.fork(0, c)
    slots, pairs = bm.append_slots([0, 1, 2, 3])
    assert pairs.tolist() == [[1, 2], [1, 3], [1, 4]]
    assert slots.tolist() == [10, 14, 18, 6]
    tables, lens = bm.export_tables([0, 1, 2, 3], 2)
    assert tables.tolist() == [[0, 2], [0, 3], [0, 4], [0, 1]] and lens.tolist() == [7] * 4


def test_block_manager_swap_and_prefix_examples(pkv):
    """The hand-worked allocator cases of the oracle, through the C++ manager."""
    bm = pkv.BlockManager(8, 4, list(range(8)), num_host_blocks=4)
    bm.add_seq(0, 6)
    bm.fork(0, 1)
    bm.add_seq(2, 3)
    assert bm.swap_out([0, 1]).tolist() == [[0, 0], [1, 1]]
    assert bm.host_refcount(0) == 2 and bm.free_list() == [3, 4, 5, 6, 7, 0, 1]
    with pytest.raises(pkv.PkvError) as e:
        bm.append_slots([0])
    assert e.value.code == pkv.PKV_ERR_INVALID
    assert bm.swap_in([1, 0]).tolist() == [[0, 3], [1, 4]]
    assert bm.refcount(3) == 2 and bm.num_host_free() == 4
    pc = pkv.BlockManager(8, 4, list(range(8)))
    p = list(range(12))
    assert pc.add_seq_tokens(0, p + [99]) == 0 and pc.num_cached_blocks() == 3
    pc.free_seq(0)
    assert pc.add_seq_tokens(1, p + [98]) == 12
    tables, _ = pc.export_tables([1], 4)
    assert tables.tolist() == [[0, 1, 2, 4]] and pc.free_list() == [5, 6, 7, 3]


def test_block_manager_decode_registration_example(pkv):
    """The hand-worked decode-registration case gives the same results in C++."""
    from tests.test_oracle_block_manager import decode_registration_example
    model = BlockManagerModel(8, 4, list(range(8)))
    cpp = pkv.BlockManager(8, 4, list(range(8)))
    assert decode_registration_example(cpp) == decode_registration_example(model)
    same_state(cpp, model)


def test_fp8_argument_errors_before_any_device_work(pkv):
    """The 8-bit entry points check shapes, paths and pointers on the host."""
    lib = pkv.library()
    fake = ctypes.c_void_p(0x1000)
    args = dict(out=fake, out_dtype=0, query=fake, kc=fake, vc=fake, ks=fake, vs=fake, tables=fake, max_blocks=4,
                lens=fake, max_ctx=64, B=2, Hq=8, Hkv=2, D=128, bs=16, NB=8, scale=0.1, part=0, path=0, ws=fake,
                ws_bytes=1 << 20)

    def call(**kw):
        a = dict(args, **kw)
        return lib.pkv_paged_attention_decode_fp8(a["out"], a["out_dtype"], a["query"], a["kc"], a["vc"], a["ks"],
                                                  a["vs"], a["tables"], a["max_blocks"], a["lens"], a["max_ctx"],
                                                  a["B"], a["Hq"], a["Hkv"], a["D"], a["bs"], a["NB"], a["scale"],
                                                  a["part"], a["path"], a["ws"], a["ws_bytes"], None, None)

    assert call(ks=None) == pkv.PKV_ERR_INVALID                  # the 8-bit pool needs its scales
    assert call(vs=None) == pkv.PKV_ERR_INVALID
    assert call(D=64) == pkv.PKV_ERR_UNSUPPORTED                 # head_dim 128 only
    assert call(Hq=2, path=pkv.PATH_TENSOR) == pkv.PKV_ERR_UNSUPPORTED   # tensor cores need grouped heads
    assert call(Hq=64, Hkv=2, path=pkv.PATH_TENSOR) == pkv.PKV_ERR_UNSUPPORTED  # group 32 > 16
    assert call(path=7) == pkv.PKV_ERR_INVALID
    assert call(ws_bytes=16) == pkv.PKV_ERR_INVALID
    assert call(B=0) == pkv.PKV_OK
    q = (fake, fake, fake, fake, fake, fake, fake)
    assert lib.pkv_reshape_and_cache_fp8(*q, 4, 8, 2, 96, 16, None, None) == pkv.PKV_ERR_UNSUPPORTED
    assert lib.pkv_reshape_and_cache_fp8(*q, 4, 8, 2, 128, 8, None, None) == pkv.PKV_ERR_UNSUPPORTED
    assert lib.pkv_reshape_and_cache_fp8(*q, 0, 8, 2, 128, 16, None, None) == pkv.PKV_OK
    assert lib.pkv_reshape_and_cache_fp8(fake, fake, fake, fake, fake, None, fake, 4, 8, 2, 128, 16, None,
                                         None) == pkv.PKV_ERR_INVALID


def test_binding_rejects_tensors_off_the_current_device(pkv, monkeypatch):
    """The binding checks devices before passing pointers: the library launches on the
    current device, so a tensor on another GPU would be a bad pointer there."""
    import types

    import torch
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)

    def fake(index, cuda=True):
        return types.SimpleNamespace(is_cuda=cuda, device=types.SimpleNamespace(index=index))

    pkv._same_device("op", fake(0), None, fake(0), fake(None, cuda=False))  # host tensors are exempt
    with pytest.raises(ValueError, match="current device cuda:0"):
        pkv._same_device("op", fake(0), fake(1))
    with pytest.raises(ValueError, match="op: every CUDA tensor"):
        pkv._same_device("op", fake(1))


def test_copy_blocks_pool_types_checked_before_device_work(pkv):
    import torch
    m = torch.zeros((1, 2), dtype=torch.int64)
    with pytest.raises(TypeError, match="bf16 or uint8"):
        pkv.copy_blocks([torch.zeros((4, 1, 16, 64))], [torch.zeros((4, 1, 16, 64))], m)
    with pytest.raises(ValueError, match="multiple of 16 bytes"):
        pkv.copy_blocks([torch.zeros((4, 1, 1, 15), dtype=torch.uint8)], [torch.zeros((4, 1, 1, 15), dtype=torch.uint8)], m)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):  # types pass, then the pointer check
        pkv.copy_blocks([torch.zeros((4, 1, 16, 64), dtype=torch.uint8)], [torch.zeros((4, 1, 16, 64), dtype=torch.uint8)], m)


def test_one_stage_ring_variant_builds_and_loads_through_the_override(pkv):
    """The build variant the ring-depth race check compares exports every declared symbol,
    and the binding loads it when PKV_LIBRARY names it (in a fresh process)."""
    import subprocess
    import sys
    from paged_kv_cache_423_b200 import build as pkv_build
    lib1 = pkv_build.build_library(variant="depth1")
    assert lib1.endswith("libpkv_depth1.so") and lib1 != pkv.library_path()
    lib = ctypes.CDLL(lib1)
    for name in declared_symbols():
        assert hasattr(lib, name), name
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = "import paged_kv_cache_423_b200 as p; p.library(); print(p.library_path()); print(p.library().pkv_version())"
    r = subprocess.run([sys.executable, "-c", code], env=dict(os.environ, PKV_LIBRARY=lib1), cwd=root,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    path, version = r.stdout.split()
    assert path == lib1 and int(version) == pkv.library().pkv_version()


def test_launch_setup_runs_once_per_device(tmp_path):
    """Kernel attributes belong to each device's context, so the launchers set them up once
    per device (csrc/per_device.h).  The bookkeeping is plain C++: compiled with g++ and run
    here, it must set each device up on first use only, keep a value per device, retry a
    failed set-up, refuse out-of-range indices, and run one set-up per device under 16 threads."""
    import shutil
    import subprocess
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    exe = tmp_path / "per_device_test"
    subprocess.run([gxx, "-std=c++17", "-O1", "-pthread", "-I", os.path.join(root, "paged_kv_cache_423_b200", "csrc"),
                    os.path.join(root, "tests", "native", "per_device_test.cpp"), "-o", str(exe)], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0 and res.stdout.strip() == "ok", res.stdout + res.stderr


def test_sequence_ids_in_any_form(pkv):
    """The allocator takes sequence ids as a list, a tuple, an int64 array (used as it is),
    an array of another integer type or any iterable; the results are the same."""
    import numpy as np
    forms = [[0, 1, 2], (0, 1, 2), np.array([0, 1, 2], np.int64), np.array([0, 1, 2], np.int32), iter([0, 1, 2]),
             {0: None, 1: None, 2: None}.keys()]
    results = []
    for ids in forms:
        bm = pkv.BlockManager(16, 4, list(range(16)))
        for s in range(3):
            bm.add_seq(s, 3 + s)
        slots, pairs = bm.append_slots(ids)
        tables, lens = bm.export_tables([0, 1, 2], 4)
        results.append((slots.tolist(), pairs.tolist(), tables.tolist(), lens.tolist()))
        bm.close()
    assert all(r == results[0] for r in results)
