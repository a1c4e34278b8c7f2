"""Benchmark of the paged decode step on B200.

One step = one decode step of one attention layer over the whole batch, i.e. every
row of the hot path:
  host block allocator (a fresh slot per sequence, CoW pairs) -> copy_blocks (when
  there are CoW pairs) -> reshape_and_cache (the new token's K/V) ->
  paged_attention_decode (plan + streaming kernel).

`value`  KV-read GB/s of the decode = sum_s L_s * Hkv * D * 2 (K and V) * 2 B per step,
         divided by the device time of the whole step, inputs resident in HBM (the
         allocator's slots/tables of every step are prepared before timing).
`e2e`    the same metric through the public API with host buffers: per step the
         allocator runs on the host, q / new K,V / slots / tables / lengths are copied
         from pinned host memory, the kernels run, and the output is read back.
`roofline` the decode call (plan + streaming kernel) against the measured HBM copy
         bandwidth, algorithmic bytes = KV + q + out + tables + lengths.

Default workload: the LLaMA-13B-shaped mixed-length batch (256 sequences, 40 heads,
head_dim 128, block size 16, lengths 70% geometric(mean 50) / 30% U{1000..2000}),
the batch on which the 70%-of-HBM target is stated.  Its KV (2.5 GB) is ~20x the
L2, so consecutive steps cannot hit in L2.  A batch whose distinct KV per step is under
4x the L2 (the shared-prefix batch) has the L2 flushed before every timed step, and
only the steps are timed.

Other rows, same JSON line (`--workload` / `--kv`):
  --kv fp8                 the same decode step over an 8-bit (e4m3) pool: KV bytes at
                           1 byte per value, reshape_and_cache_fp8 + paged_attention_decode_fp8.
  --workload chunked_prefill_13b | chunked_prefill_long_gqa
                           one step = the chunks' K/V written + paged_attention_prefill;
                           value in TFLOP/s (4 * D per visible (row, key) per head),
                           roofline against the measured bf16 tensor peak.
  --workload prefix_beams [--beams 4]
                           128 sequences sharing one 1024-token prompt (the prompt's blocks
                           in every table); with --beams N each is first forked into N beams,
                           so the first step copies every shared partial last block but one.
                           The decode is the shared-prefix decode (the allocator's tables
                           planned on the host once per step; --shared off for the plain one).
  --workload swap_llama13b one step = 256 13B-shaped blocks swapped out to pinned host
                           memory and 256 swapped in (K and V); GB/s against the
                           pinned-memory copy bandwidth measured in the same run.

`--impl reference` times the CPU oracle (float64 NumPy, one thread) on a bounded
sample of the same workload and prints the same JSON line with "impl": "reference".
Multi-GPU (`torchrun`): independent replicas per GPU (weak scaling), no collective on
the data path; timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "paged decode attention KV-read GB/s (% of B200 HBM peak); seq-steps/sec"
METRIC_PREFILL = "paged prefill attention TFLOP/s (% of B200 bf16 tensor peak)"
METRIC_SWAP = "swap_blocks device<->pinned-host GB/s (% of the pinned memcpy bandwidth)"
SWAP_WORKLOAD = "swap_llama13b"
FALLBACK_HBM_GBS = 6650.0


def measured_bf16_tflops():
    """The sustained cuBLAS bf16 figure: the prefill kernel is timed inside a loop of
    back-to-back launches lasting seconds."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured (sustained)"
    except Exception:
        return 1400.0, "fallback (sustained)"


def measured_hbm_gbs():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# Sources each profiled kernel is compiled from: a recorded ncu traffic figure is only
# reported while these files are the ones it was measured on.
KERNEL_SOURCES = {
    "decode_simt": ["decode.cu", "decode_common.cuh", "device_common.cuh"],
    "decode_gqa_tc": ["decode_gqa_tc.cu", "decode_common.cuh", "device_common.cuh", "tcgen05_common.cuh"],
    "decode_gqa_tc_fp8": ["decode_gqa_tc_fp8.cu", "decode_common.cuh", "device_common.cuh", "tcgen05_common.cuh"],
    "prefill": ["prefill_tc.cu", "decode_common.cuh", "device_common.cuh", "tcgen05_common.cuh"],
    "shared": ["shared_decode.cu", "shared_plan.cpp", "prefill_tc.cu", "decode_gqa_tc.cu", "decode.cu",
               "decode_common.cuh", "device_common.cuh", "tcgen05_common.cuh"],
    "shared_fp8": ["shared_decode.cu", "shared_plan.cpp", "prefill_tc.cu", "decode_gqa_tc_fp8.cu", "decode_gqa_tc.cu",
                   "decode.cu", "decode_common.cuh", "device_common.cuh", "tcgen05_common.cuh"],
}


def source_digest(kind: str) -> str:
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "paged_kv_cache_423_b200", "csrc")
    for f in KERNEL_SOURCES[kind]:
        h.update(f.encode())
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(key: str, kind: str, units: int, layout=None):
    """DRAM bytes (read + write) per launch of the profiled kernel from profiles/traffic.json, or
    None unless the entry was captured on the same kernel sources, the same table layout and a
    batch of the same size: `units` (the algorithmic bytes, or flops, of one launch) within 5% of
    the capture's.  Contexts grow by a token per step, so a run with another step count has a
    slightly different mean; the recorded bytes are scaled by the ratio of the units."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            entry = json.load(f).get(key)
    except Exception:
        return None
    if not entry or entry.get("sources") != source_digest(kind) or entry.get("layout") != layout:
        return None
    rec = entry.get("algorithmic_per_launch")
    if not rec or abs(int(units) - rec) > 0.05 * rec:
        return None
    return int(round(entry["dram_bytes_per_launch"] * int(units) / rec))


SPEC_HBM_GBS = 8000.0  # B200 HBM3e nominal (DGX figure)
# The shared-prefix decode's private phase runs on the CUDA-core decode when no row's remainder
# is longer than this (one 128-token tile), else on the tensor-core decode (csrc/shared_decode.cu).
SHARED_SIMT_SUFFIX_MAX = 128
L2_BYTES = 126 * 1000 ** 2  # B200 L2


# The length mixes the batches are drawn with (workloads.draw_lengths), recorded in each line.
LENGTH_MIX = {
    "tiny": "{1, 7, 16, 33}",
    "llama7b": "U{10..2000}",
    "llama13b_mixed_bs16": "70% geometric(mean 50), 30% U{1000..2000}",
    "llama13b_mixed_bs32": "70% geometric(mean 50), 30% U{1000..2000}",
    "prefix_beams": f"{wl.PREFIX_TOKENS}-token shared prompt + U{{10..500}}",
    "long_trace": "U{5000..32000} (a static batch)",
}


def needs_l2_flush(distinct_bytes_per_step: int) -> bool:
    """Steps whose distinct KV is under 4x the L2 could be served partly from what the
    previous step left there, so the timed loop flushes the L2 between them."""
    return distinct_bytes_per_step < 4 * L2_BYTES


def stream_read_gbs(pkv, device, nbytes=4 << 30, reps=10):
    """HBM read bandwidth reached in this run by the library's read-only streaming
    kernel over a buffer 32x the L2 (so nothing is served from L2), CUDA events on the
    current stream after 3 warm-up passes.  The roofline's second denominator."""
    import torch
    buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
    sink = torch.zeros(1, dtype=torch.int32, device=device)
    for _ in range(3):
        pkv.stream_read(buf, sink)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(reps):
        pkv.stream_read(buf, sink)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    del buf
    return nbytes * reps / (ms * 1e-3) / 1e9


def split_tokens(num_seqs, num_kv_heads, block_size, max_context_len, tensor):
    """The library's automatic split of a context (tokens per partition) for a call:
    the CUDA-core path takes the largest of 512..64 that leaves >= 16384 work items,
    the tensor-core paths the largest of 2048.. down to that which leaves >= 8 items
    per SM, and not below 512 with at least 4 (sequence, kv head) units per SM.  Used
    to count the launches of a step (a split context adds the merge)."""
    def items(p):
        return num_seqs * num_kv_heads * -(-max_context_len // p)
    base = 512
    while base > 64 and items(base) < 16384:
        base //= 2
    base = max(base, block_size)
    if not tensor:
        return base
    p = 2048
    while p > base and items(p) < 8 * 148:
        p //= 2
    if num_seqs * num_kv_heads >= 4 * 148 and p < 512:
        p = 512
    return max(p, base)


def rank_info():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


# ---------------------------------------------------------------------------
# clocks sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """Samples the SM clock and the clock-event reasons through NVML back to back (a
    pause of 0.2 ms between samples) while the timed region runs (a thread; NVML reads
    only, nothing is set).  Entering waits for the first sample, so a timed region of a
    few milliseconds still gets several."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, torch_device):
        self.dev = torch_device
        self.samples = []
        self.max_mhz = None
        self.err = None
        self._stop = None
        self._thread = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            p = torch.cuda.get_device_properties(self.dev)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.dev.index or 0)

    def __enter__(self):
        import threading
        try:
            import pynvml
            h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: record why
            self.err = f"nvml unavailable: {e}"
            return self
        self._stop = threading.Event()

        def poll():
            while not self._stop.is_set():
                try:
                    mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((mhz, rs))
                except Exception as e:
                    self.err = str(e)
                    return
                time.sleep(0.0002)

        self._thread = threading.Thread(target=poll, daemon=True)
        self._thread.start()
        t0 = time.perf_counter()
        while not self.samples and self.err is None and time.perf_counter() - t0 < 1.0:
            time.sleep(0.0001)
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [self.err or "no samples"], "samples": 0}
        mhz = [m for m, _ in self.samples]
        reasons = sorted({name for _, rs in self.samples for name, bit in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples), "sm_mhz_min": min(mhz)}


# ---------------------------------------------------------------------------
# Workload preparation (allocator + per-step inputs)
# ---------------------------------------------------------------------------

def decode_bytes(lens, Hq, Hkv, D, bs, kv_elem_bytes=2):
    """Algorithmic bytes of one decode call: KV of every valid token once, q, out (bf16),
    the used table entries and the lengths."""
    lens = np.asarray(lens, np.int64)
    kv = int(lens.sum()) * Hkv * D * 2 * kv_elem_bytes
    blocks = int(np.sum(-(-lens // bs)))
    return kv, kv + 2 * len(lens) * Hq * D * 2 + blocks * 4 + len(lens) * 4


def unique_kv_bytes(tables, lens, Hkv, D, bs, kv_elem_bytes=2):
    """KV bytes of one decode call with every physical block counted once: for each
    distinct block, the rows any sequence reads from it (a shared prefix block is read
    through many tables but holds its bytes once)."""
    tables = np.asarray(tables)
    lens = np.asarray(lens, np.int64)
    rows = np.zeros(int(tables.max()) + 1 if tables.size else 1, np.int64)
    for s, L in enumerate(lens):
        need = -(-int(L) // bs)
        if need == 0:
            continue
        r = np.full(need, bs, np.int64)
        if L % bs:
            r[-1] = L % bs
        np.maximum.at(rows, tables[s][:need].astype(np.int64), r)
    return int(rows.sum()) * Hkv * D * 2 * kv_elem_bytes


def e4m3_pool(shape, gen, device):
    """Seeded e4m3 codes drawn as bit patterns on the device (sign, exponent around 8,
    uniform mantissa, never NaN), like workloads.e4m3_codes."""
    import torch
    sign = torch.randint(0, 2, shape, generator=gen, device=device, dtype=torch.int32)
    exp = (torch.randn(shape, generator=gen, device=device) * 1.5 + 8).round().clamp(0, 15).to(torch.int32)
    mant = torch.randint(0, 8, shape, generator=gen, device=device, dtype=torch.int32)
    mant = torch.where((exp == 15) & (mant == 7), torch.full_like(mant, 6), mant)
    return ((sign << 7) | (exp << 3) | mant).to(torch.uint8)


class ModelManager:
    """The allocator's reference model (`oracle.block_manager.BlockManagerModel`) with the
    C++ manager's array outputs.  The reference arm builds its tables with it, so that it
    loads nothing from the library; the operations are the same, so the tables are too."""

    def __init__(self, num_blocks, block_size, initial_order=None):
        from oracle.block_manager import BlockManagerModel
        self.m = BlockManagerModel(num_blocks, block_size, initial_order=initial_order)

    def add_seq(self, seq_id, num_tokens, shared_prefix_blocks=()):
        self.m.add_seq(seq_id, num_tokens, [int(b) for b in shared_prefix_blocks])

    def fork(self, parent, child):
        self.m.fork(parent, child)

    def append_slots(self, seq_ids):
        slots, pairs = self.m.append_slots([int(s) for s in seq_ids])
        return np.asarray(slots, np.int64), np.asarray(pairs, np.int64).reshape(-1, 2)

    def slots(self, seq_id, start, count):
        return np.asarray(self.m.slots(seq_id, start, count), np.int64)

    def export_tables(self, seq_ids, max_blocks):
        ids = [int(s) for s in seq_ids]
        tables, lens = self.m.export_tables(ids, max_blocks)
        return np.asarray(tables, np.int32).reshape(len(ids), max_blocks), np.asarray(lens, np.int32)

    def num_free(self):
        return self.m.num_free()

    def refcount(self, b):
        return self.m.refcount(b)

    def close(self):
        pass


class Workload:
    def __init__(self, name: str, steps: int, seed: int, device, kv8: bool = False, beams: int = 1,
                 native: bool = True):
        """native=False (the reference arm): the library is not loaded and the batch's
        tables come from the allocator's reference model."""
        import torch
        if native:
            import paged_kv_cache_423_b200 as pkv
        else:
            pkv = None
        self.name = name
        self.kv8 = kv8
        self.beams = beams
        b = wl.make_decode_batch(name, with_data=False, extra_blocks=0)
        self.parents = b.num_seqs
        self.B, self.Hq, self.Hkv, self.D, self.bs = b.num_seqs * beams, b.num_heads, b.num_kv_heads, b.head_dim, b.block_size
        self.seq_ids = np.asarray(beam_ids(self.parents, beams), np.int64)  # row order of every step's tensors
        self.scale = b.scale
        self.parent_lens0 = b.context_lens.copy()
        self.lens0 = np.repeat(b.context_lens, beams)  # per row: context length after the first appended token
        growth = steps + 1
        need_final = int(np.sum(-(-(self.lens0 + growth) // self.bs)))
        self.NB = max(b.num_blocks, int(math.ceil(1.2 * need_final)))
        self.free_order = wl.rng_for(seed).permutation(self.NB).astype(np.int32)
        self.max_blocks = int(np.max(-(-(self.lens0 + growth) // self.bs)))
        self.device = device
        self.pkv = pkv
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        shape = (self.NB, self.Hkv, self.bs, self.D)
        if kv8:
            self.key_cache = e4m3_pool(shape, g, device)
            self.value_cache = e4m3_pool(shape, g, device)
            srng = wl.rng_for(seed + 2)
            self.k_scale = torch.from_numpy(wl.kv_scales(srng, self.Hkv)).to(device)
            self.v_scale = torch.from_numpy(wl.kv_scales(srng, self.Hkv)).to(device)
        else:
            self.key_cache = torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
            self.value_cache = torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
        self.rng = wl.rng_for(seed + 1)
        # the shared-prefix batch: one copy of the prompt's blocks in every table
        self.shared_blocks = wl.PREFIX_TOKENS // self.bs if name == "prefix_beams" else 0
        self.layout = f"shared prompt: {self.shared_blocks} blocks in every table" if self.shared_blocks else None
        if beams > 1:
            self.layout = (self.layout + "; " if self.layout else "") + f"{beams} beams forked from every sequence"
        self.label = name + (f"+beams{beams}" if beams > 1 else "") + ("+fp8" if kv8 else "")

    def write(self, k, v, slots, status):
        if self.kv8:
            self.pkv.reshape_and_cache_fp8(k, v, self.key_cache, self.value_cache, slots, self.k_scale, self.v_scale,
                                           status=status)
        else:
            self.pkv.reshape_and_cache(k, v, self.key_cache, self.value_cache, slots, status=status)

    def copy(self, pairs, status):
        self.pkv.copy_blocks([self.key_cache], [self.value_cache], pairs, status=status)

    def decode(self, out, q, tables, lens, max_len, ws, path, status, shared=None):
        """shared = (device plan, its info, the shared-prefix workspace) for the shared-prefix decode."""
        if shared is not None and self.kv8:
            plan, info, sws = shared
            self.pkv.paged_attention_decode_shared_fp8(out, q, self.key_cache, self.value_cache, self.k_scale,
                                                       self.v_scale, tables, lens, self.scale, plan, info, sws,
                                                       status=status)
        elif shared is not None:
            plan, info, sws = shared
            self.pkv.paged_attention_decode_shared(out, q, self.key_cache, self.value_cache, tables, lens, self.scale,
                                                   plan, info, sws, status=status)
        elif self.kv8:
            self.pkv.paged_attention_decode_fp8(out, q, self.key_cache, self.value_cache, self.k_scale, self.v_scale,
                                                tables, lens, max_len, self.scale, ws, path=path, status=status)
        else:
            self.pkv.paged_attention_decode(out, q, self.key_cache, self.value_cache, tables, lens, max_len, self.scale,
                                            ws, path=path, status=status)

    def new_manager(self):
        factory = self.pkv.BlockManager if self.pkv is not None else ModelManager
        return build_manager(factory, self.NB, self.bs, self.free_order, self.parent_lens0 - 1, self.shared_blocks,
                             self.max_blocks, self.beams)

    def host_step_inputs(self):
        q = wl.bf16_normal(self.rng, (self.B, self.Hq, self.D))
        k, v = wl.new_tokens(self.rng, self.B, self.Hkv, self.D)
        return q, k, v


def shared_min_rows(args) -> int:
    """Fewest rows a shared segment serves.  Over a bf16 pool a segment of 2 rows already saves
    reads; over an 8-bit pool a segment's blocks are first widened to bf16 scratch (a read of the
    codes, a write and a read of twice their bytes), which costs more than 4 rows reading the
    codes themselves: there segments start at 5 rows (4-beam batch: 0.139 against 0.175 ms per
    call with 4-row segments; 0.185 against 0.136 ms the other way round over bf16)."""
    mr = getattr(args, "min_rows", None)
    return mr if mr is not None else (5 if getattr(args, "kv", "bf16") == "fp8" else 2)


def shared_decode_applies(args, w) -> bool:
    """The shared-prefix decode: on request, or by default for the shared-prompt workload;
    it needs the tensor-core decode's head shapes (bf16 or 8-bit pool)."""
    g = w.Hq // w.Hkv
    ok = w.D == 128 and 2 <= g <= 16 and args.path != "simt"
    choice = getattr(args, "shared", "auto")
    if choice == "on" and not ok:
        raise SystemExit("--shared on needs head_dim 128 and 2 <= num_heads / num_kv_heads <= 16")
    return ok and (choice == "on" or (choice == "auto" and w.shared_blocks > 0))


def beam_ids(parents: int, beams: int) -> list:
    """Row order of a batch of `parents` sequences with `beams` beams each: every parent
    id followed by its children (ids parents + (beams - 1) * s + k).  Appends in this
    order give a shared partial last block a copy for every beam but the last, which
    writes in place."""
    ids = []
    for s in range(parents):
        ids.append(s)
        ids.extend(parents + (beams - 1) * s + k for k in range(beams - 1))
    return ids


def build_manager(new_manager, num_blocks, bs, free_order, lens, shared_blocks, max_blocks, beams=1):
    """The batch in an allocator made by `new_manager(num_blocks, bs, free_order)` (the C++
    `BlockManager`, or `ModelManager` for the reference arm): sequence s holds lens[s] tokens; with
    shared_blocks = P, sequence 0's first P blocks (one system prompt) are also the
    first P blocks of every other table (reference count B), the rest private; with
    beams > 1 every sequence is then forked into that many beams (`beam_ids`)."""
    bm = new_manager(num_blocks, bs, free_order)
    prefix = ()
    for s in range(len(lens)):
        bm.add_seq(s, int(lens[s]), prefix)
        if s == 0 and shared_blocks:
            prefix = bm.export_tables([0], max_blocks)[0][0, :shared_blocks].tolist()
    parents = len(lens)
    for s in range(parents):
        for k in range(beams - 1):
            bm.fork(s, parents + (beams - 1) * s + k)
    return bm


def pool_usage(num_blocks: int, num_free: int, lens, bs: int) -> dict:
    """Pool blocks in use against the blocks the tables reference (each table's view);
    sharing shows as `saved_by_sharing` > 0."""
    referenced = int(np.sum(-(-np.asarray(lens, np.int64) // bs)))
    used = num_blocks - num_free
    return {"blocks": num_blocks, "used": used, "utilisation": round(used / num_blocks, 4),
            "referenced_by_tables": referenced,
            "saved_by_sharing": round(1 - used / referenced, 4) if referenced else 0.0}


def aggregate_over_ranks(ms_local, units_local, dist=None, device=None):
    """Whole-job timing: the slowest rank's time and the units all ranks processed.

    Every rank must call this with the same collective sequence (MAX then SUM)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(ms_local), int(units_local)
    import torch
    t = torch.tensor([float(ms_local)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    u = torch.tensor([int(units_local)], dtype=torch.int64, device=device)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), int(u.item())


def to_dev(bits, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bench_device(local_rank: int):
    """The CUDA device of this rank (one process per GPU)."""
    import torch
    return torch.device(f"cuda:{local_rank}")


def run_ours(args, rank, world, local_rank):
    import torch
    import paged_kv_cache_423_b200 as pkv

    device = bench_device(local_rank)
    torch.cuda.set_device(device)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=device)
    total = args.warmup + args.steps
    n_states = min(total, args.states)
    kv8 = args.kv == "fp8"
    w = Workload(args.workload, max(n_states, min(total, args.e2e_steps + args.warmup)), seed=1000 + rank,
                 device=device, kv8=kv8, beams=args.beams)
    seq_ids = w.seq_ids

    # ---- the allocator runs ahead of timing: `n_states` consecutive decode steps of
    # the batch.  Timed step i replays state i % n_states, so the batch keeps its
    # configured length mix however many steps are timed (a replayed state rewrites
    # its own token into its own slot, then decodes the same contexts).
    g = w.Hq // w.Hkv
    use_shared = shared_decode_applies(args, w)
    bm = w.new_manager()
    states = []
    for _ in range(n_states):
        slots, pairs = bm.append_slots(seq_ids)
        tables, lens = bm.export_tables(seq_ids, w.max_blocks)
        q, k, v = w.host_step_inputs()
        plan = None
        if use_shared:
            plan_h, info = pkv.shared_plan(tables, lens, w.Hq, w.Hkv, w.bs, min_rows=shared_min_rows(args),
                                           key_chunk=getattr(args, "key_chunk", 0))
            plan = (torch.from_numpy(plan_h).to(device), info)
        states.append(dict(plan=plan, q=to_dev(q, device), k=to_dev(k, device), v=to_dev(v, device),
                           slots=torch.from_numpy(slots).to(device), pairs=torch.from_numpy(pairs).to(device),
                           n_pairs=len(pairs), tables=torch.from_numpy(tables).to(device),
                           lens=torch.from_numpy(lens).to(device), max_len=int(lens.max()), host_lens=lens,
                           unique_kv=unique_kv_bytes(tables, lens, w.Hkv, w.D, w.bs, 1 if kv8 else 2)))
    pool = pool_usage(w.NB, bm.num_free(), lens, w.bs)  # after the last prepared step
    bm.close()
    max_len_all = int(w.lens0.max()) + max(n_states, args.e2e_steps + args.warmup) + 1
    ws = torch.empty(pkv.paged_attention_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.bs, max_len_all),
                     dtype=torch.uint8, device=device)
    out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream()
    path = {"auto": 0, "simt": 1, "tensor": 2}[args.path]
    sws = None
    if use_shared:
        size_fn = (pkv.paged_attention_decode_shared_fp8_workspace_size if kv8
                   else pkv.paged_attention_decode_shared_workspace_size)
        sws = torch.empty(max(size_fn(st["plan"][1], w.Hq, w.Hkv, w.D) for st in states), dtype=torch.uint8,
                          device=device)

    def step(i, ev=None):
        st = states[i % n_states]
        if st["n_pairs"]:
            w.copy(st["pairs"], status)
        w.write(st["k"], st["v"], st["slots"], status)
        if ev is not None:
            ev[0].record(stream)
        w.decode(out, st["q"], st["tables"], st["lens"], max_len_all, ws, path, status,
                 shared=(st["plan"][0], st["plan"][1], sws) if use_shared else None)
        if ev is not None:
            ev[1].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    launches = 0
    kv_total = bytes_total = unique_total = unique_kv_total = 0
    uses_tensor = path == 2 or (path == 0 and w.D == 128 and 2 <= g <= 16)
    # write, plan, decode (+ copy_blocks when a fork copied blocks) (+ the merge of a split context)
    merge = 1 if uses_tensor and max_len_all > split_tokens(w.B, w.Hkv, w.bs, max_len_all, True) else 0
    for i in range(args.warmup, total):
        st = states[i % n_states]
        kv, alg = decode_bytes(st["host_lens"], w.Hq, w.Hkv, w.D, w.bs, 1 if kv8 else 2)
        kv_total += kv
        bytes_total += alg
        unique_total += alg - kv + st["unique_kv"]
        unique_kv_total += st["unique_kv"]
        if use_shared:  # write, setup, [widening and] shared phase (when there are segments), plan,
            # [query split (8-bit tensor-core private phase),] decode, merge
            info = st["plan"][1]
            launches += (5 + (1 if info.num_entries else 0) * (2 if kv8 else 1)
                         + (1 if kv8 and info.max_suffix_len > SHARED_SIMT_SUFFIX_MAX else 0)
                         + (1 if st["n_pairs"] else 0))
        else:
            launches += 3 + (1 if st["n_pairs"] else 0) + merge
    dec_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush_l2 = needs_l2_flush(min(st["unique_kv"] for st in states))
    if flush_l2:  # a write of 2x the L2 before each step; only the steps are timed
        flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)
        step_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(device) as clocks:
        t0.record(stream)
        for j, i in enumerate(range(args.warmup, total)):
            if flush_l2:
                flush_buf.fill_(j & 0xff)
                step_events[j][0].record(stream)
            step(i, dec_events[j])
            if flush_l2:
                step_events[j][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ms = sum(a.elapsed_time(b) for a, b in step_events) if flush_l2 else t0.elapsed_time(t1)
    dec_ms = sum(a.elapsed_time(b) for a, b in dec_events)
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item():#x}")
    ms_max, kv_all = aggregate_over_ranks(ms, kv_total, dist, device)
    value = kv_all / (ms_max * 1e-3) / 1e9
    seq_steps = world * w.B * args.steps / (ms_max * 1e-3)

    # ---- e2e through the public API with host buffers
    e2e = run_e2e(args, w, pkv, device, path, ws, out, status, max_len_all, sws) if not args.no_e2e else None

    peak, peak_kind = measured_hbm_gbs()
    # the roofline counts every physical block once (a shared prefix is one copy of bytes);
    # the same as the logical count when no blocks are shared
    dec_gbs = unique_total / (dec_ms * 1e-3) / 1e9
    read_gbs = stream_read_gbs(pkv, device)
    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 KV, bf16 q" if kv8 else "bf16", "data": "synthetic",
        "config": {"workload": w.label, "kv_dtype": args.kv, "num_seqs": w.B, "beams": w.beams, "num_heads": w.Hq, "num_kv_heads": w.Hkv, "head_dim": w.D,
                   "block_size": w.bs, "lengths": LENGTH_MIX[w.name], "mean_context": float(np.mean(w.lens0)),
                   "num_blocks": w.NB, "pool": pool,
                   "kv_bytes_per_step": kv_total // args.steps, "path": args.path,
                   "decode": "shared-prefix" if use_shared else "plain",
                   **({"shared_min_rows": shared_min_rows(args)} if use_shared else {}),
                   "l2": ("L2 flushed before each timed step (a 252 MB write, outside the step's events): the"
                          " distinct KV per step is under 4x the 126 MB L2; e2e steps are pipelined, not flushed"
                          if flush_l2 else "inputs larger than L2 (distinct KV per step >= 4x the 126 MB L2)"),
                   "parallelism": f"replicas{world}" if world > 1 else "single"},
        "seq_steps_per_s": round(seq_steps, 1),
        "seq_steps_per_s_decode_call": round(w.B * args.steps / (dec_ms * 1e-3), 1),
        # of the HBM peak, on distinct KV bytes (a shared block's bytes once; the same as
        # `value` unless tables share blocks, when logical GB/s can exceed the peak)
        "pct_hbm_peak": round(100 * value * (unique_kv_total / kv_total if kv_total else 1.0) / world / peak, 2),
        "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(dec_gbs / peak, 4),
                     "traffic": recorded_traffic(w.label + ("+shared" if use_shared else ""),
                                                 ("shared_fp8" if kv8 else "shared") if use_shared else
                                                 ("decode_gqa_tc_fp8" if kv8 else "decode_gqa_tc") if uses_tensor
                                                 else "decode_simt", unique_total // args.steps, w.layout),
                     "algorithmic_bytes_per_launch": unique_total // args.steps,
                     "logical_bytes_per_launch": bytes_total // args.steps, "peak_kind": peak_kind,
                     "kernel": ("paged_attention_decode_shared_fp8: setup + shared phase (the shared blocks widened"
                                " to bf16, tcgen05 prefill kernel, every key visible, partials) + plan + decode of"
                                " the private remainders (CUDA cores when none passes 128 tokens, else query split +"
                                " tcgen05 kind::f8f6f4) + merge; traffic = the DRAM bytes of all of them"
                                if use_shared and kv8
                                else "paged_attention_decode_shared: setup + shared phase (tcgen05 prefill kernel, every"
                                " key visible, partials) + plan + decode of the private remainders (CUDA cores when"
                                " none passes 128 tokens, else tcgen05) + merge; traffic = the DRAM bytes of all of"
                                " them" if use_shared
                                else "paged_attention_decode_fp8: plan + tcgen05 kind::f8f6f4 kernel on the e4m3 tiles"
                                " + split merge" if kv8 and uses_tensor
                                else "paged_attention_decode_fp8: plan + CUDA-core streaming kernel (e4m3 tiles)" if kv8
                                else "paged_attention_decode: plan + tcgen05 kernel + split merge" if uses_tensor
                                else "paged_attention_decode: plan + CUDA-core streaming kernel"),
                     "ms_per_launch": round(dec_ms / args.steps, 4),
                     "ms_per_launch_median": round(statistics.median(a.elapsed_time(b) for a, b in dec_events), 4),
                     # the same achieved figure against the other two denominators
                     "peaks_gbs": {f"copy_{peak_kind}": peak, "read_stream_in_run": round(read_gbs, 1),
                                   "spec": SPEC_HBM_GBS},
                     "frac_of": {f"copy_{peak_kind}": round(dec_gbs / peak, 4),
                                 "read_stream_in_run": round(dec_gbs / read_gbs, 4),
                                 "spec": round(dec_gbs / SPEC_HBM_GBS, 4)}},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    if e2e is not None:
        result["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not kv8:
        result["cpu_baseline"] = cpu_baseline(w, states[0], budget_s=args.cpu_budget)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and kv8:
        result["cpu_baseline"] = cpu_baseline_fp8(w, states[0], budget_s=args.cpu_budget)
    if dist:
        dist.destroy_process_group()
    return result


def run_e2e(args, w, pkv, device, path, ws, out, status, max_len_bound, sws=None):
    """End to end through the public API with host buffers, pipelined as a server
    would run it: per step the C++ allocator produces slots and tables on the host;
    q, new K, new V (one pinned buffer per step) go host->device on a copy stream as soon
    as the step before has been launched (beside its kernels), and the allocator output
    (a small pinned buffer, double-buffered) once the allocator has run; the step's
    output comes back to pinned memory on a stream of its own (beside the next step's
    kernels) and is read on the host two steps later (outputs triple-buffered), so the
    host never waits for the step that runs while it prepares the next.  Every timed
    step's copies are issued inside the timed region.  With the shared-prefix decode (`sws` its workspace)
    the host also plans each step from the allocator's tables, and the plan travels with
    them."""
    import torch
    ke = max(1, min(args.steps, args.e2e_steps))
    n = args.warmup + ke
    bm = w.new_manager()
    seq_ids = w.seq_ids
    compute = torch.cuda.current_stream()
    copy = torch.cuda.Stream(device=device)
    d2h = torch.cuda.Stream(device=device)          # results back to the host beside the next step
    nq, nk = w.B * w.Hq * w.D, w.B * w.Hkv * w.D
    # per-step pinned q | k | v (bf16 bits)
    host_qkv = []
    for _ in range(n):
        q, k, v = w.host_step_inputs()
        host_qkv.append(torch.from_numpy(np.concatenate([q.ravel(), k.ravel(), v.ravel()]).view(np.int16)).pin_memory())
    # allocator output: slots (int64) | pairs (int64 x2) | tables (int32) | lens (int32), 256-byte aligned parts
    def al(x):
        return (x + 255) // 256 * 256
    o_slots, o_pairs = 0, al(8 * w.B)
    o_tab = o_pairs + al(16 * w.B)
    o_lens = o_tab + al(4 * w.B * w.max_blocks)
    o_plan = o_lens + al(4 * w.B)
    plan_cap = 0
    if sws is not None:  # room for the largest plan and workspace: sized on a dry run of the allocator
        size_fn = (pkv.paged_attention_decode_shared_fp8_workspace_size if w.kv8
                   else pkv.paged_attention_decode_shared_workspace_size)
        ws_need = sws.numel()
        probe = w.new_manager()
        for _ in range(n):
            probe.append_slots(seq_ids)
            t_, l_ = probe.export_tables(seq_ids, w.max_blocks)
            info_ = pkv.shared_plan(t_, l_, w.Hq, w.Hkv, w.bs, min_rows=shared_min_rows(args),
                                    key_chunk=getattr(args, "key_chunk", 0))[1]
            plan_cap = max(plan_cap, int(info_.bytes))
            ws_need = max(ws_need, size_fn(info_, w.Hq, w.Hkv, w.D))
        probe.close()
        if ws_need > sws.numel():  # the e2e run goes further than the timed steps' states
            sws = torch.empty(ws_need, dtype=torch.uint8, device=device)
    meta_bytes = o_plan + al(plan_cap)
    host_meta = [torch.empty(meta_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]
    dev_qkv = [torch.empty(nq + 2 * nk, dtype=torch.int16, device=device) for _ in range(2)]
    dev_meta = [torch.empty(meta_bytes, dtype=torch.uint8, device=device) for _ in range(2)]
    out_host = [torch.empty(out.shape, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    outs = [out, torch.empty_like(out), torch.empty_like(out)]
    h2d_done = [torch.cuda.Event() for _ in range(n)]
    qkv_done = [torch.cuda.Event() for _ in range(n)]
    comp_done = [torch.cuda.Event() for _ in range(n)]
    d2h_done = [torch.cuda.Event() for _ in range(n)]
    stats = {"h2d": 0, "d2h": 0, "kv": 0, "checksum": 0.0, "host_s": 0.0}
    # the step's device views, made once per buffer (the host loop is part of what is timed)
    views = []
    for b in range(2):
        dm = dev_meta[b]
        views.append({"q": dev_qkv[b][:nq].view(torch.bfloat16).view(w.B, w.Hq, w.D),
                      "k": dev_qkv[b][nq:nq + nk].view(torch.bfloat16).view(w.B, w.Hkv, w.D),
                      "v": dev_qkv[b][nq + nk:].view(torch.bfloat16).view(w.B, w.Hkv, w.D),
                      "slots": dm[o_slots:o_slots + 8 * w.B].view(torch.int64),
                      "tables": dm[o_tab:o_tab + 4 * w.B * w.max_blocks].view(torch.int32).view(w.B, w.max_blocks),
                      "lens": dm[o_lens:o_lens + 4 * w.B].view(torch.int32),
                      "plan": dm[o_plan:o_plan + plan_cap]})

    def upload_qkv(i):
        """Step i's q, new K and new V to the device, once step i-2 is done with the buffer."""
        with torch.cuda.stream(copy):
            if i >= 2:
                copy.wait_event(comp_done[i - 2])
            dev_qkv[i % 2].copy_(host_qkv[i], non_blocking=True)
            qkv_done[i].record(copy)

    def step(i, prefetch_next):
        b = i % 2
        t_in = time.perf_counter()
        wait_s = 0.0
        if i >= 2:
            tw = time.perf_counter()
            h2d_done[i - 2].synchronize()          # host_meta[b] is free again
            wait_s += time.perf_counter() - tw
        slots, pairs = bm.append_slots(seq_ids)
        tables, lens = bm.export_tables(seq_ids, w.max_blocks)
        hm = host_meta[b].numpy()
        hm[o_slots:o_slots + slots.nbytes] = slots.view(np.uint8)
        hm[o_tab:o_tab + tables.nbytes] = tables.reshape(-1).view(np.uint8)
        hm[o_lens:o_lens + lens.nbytes] = lens.view(np.uint8)
        if len(pairs):
            hm[o_pairs:o_pairs + pairs.nbytes] = pairs.reshape(-1).view(np.uint8)
        plan_bytes = 0
        if sws is not None:  # planned straight into the pinned buffer (raises if it outgrew it)
            plan_h, info = pkv.shared_plan(tables, lens, w.Hq, w.Hkv, w.bs, min_rows=shared_min_rows(args),
                                           key_chunk=getattr(args, "key_chunk", 0), out=hm[o_plan:o_plan + plan_cap])
            plan_bytes = plan_h.nbytes
        with torch.cuda.stream(copy):
            if i >= 2:
                copy.wait_event(comp_done[i - 2])  # device buffers b are free again
            dev_meta[b].copy_(host_meta[b], non_blocking=True)
            h2d_done[i].record(copy)
        compute.wait_event(qkv_done[i])
        compute.wait_event(h2d_done[i])
        vw = views[b]
        if len(pairs):
            d_pairs = dev_meta[b][o_pairs:o_pairs + pairs.nbytes].view(torch.int64).view(-1, 2)
            w.copy(d_pairs, status)
        w.write(vw["k"], vw["v"], vw["slots"], status)
        r = i % 3                                  # output buffers
        if i >= 3:
            compute.wait_event(d2h_done[i - 3])    # outs[r] has been copied out
        shared = (vw["plan"], info, sws) if sws is not None else None
        w.decode(outs[r], vw["q"], vw["tables"], vw["lens"], max_len_bound, ws, path, status, shared=shared)
        comp_done[i].record(compute)
        with torch.cuda.stream(d2h):
            d2h.wait_event(comp_done[i])
            out_host[r].copy_(outs[r], non_blocking=True)
            d2h_done[i].record(d2h)
        if prefetch_next:                          # the next step's inputs go up beside this step's kernels
            upload_qkv(i + 1)
        if i >= 2:                                 # read the result of two steps back on the host
            tw = time.perf_counter()
            d2h_done[i - 2].synchronize()
            wait_s += time.perf_counter() - tw
            stats["checksum"] += float(out_host[(i - 2) % 3][0, 0, 0])
        if i >= args.warmup:
            stats["host_s"] += time.perf_counter() - t_in - wait_s
            stats["h2d"] += (host_qkv[i].numel() * 2 + slots.nbytes + pairs.nbytes + tables.nbytes + lens.nbytes
                             + plan_bytes)
            stats["d2h"] += out_host[r].numel() * 2
            stats["kv"] += int(np.asarray(lens, np.int64).sum()) * w.Hkv * w.D * 2 * (1 if w.kv8 else 2)

    if args.warmup > 0:
        upload_qkv(0)
    for i in range(args.warmup):
        step(i, prefetch_next=i + 1 < args.warmup)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(copy)
    compute.wait_event(t0)
    upload_qkv(args.warmup)                        # the first timed step's inputs, inside the timed region
    for i in range(args.warmup, n):
        step(i, prefetch_next=i + 1 < n)
    for j in range(max(0, n - 2), n):              # the last two steps' results
        d2h_done[j].synchronize()
        stats["checksum"] += float(out_host[j % 3][0, 0, 0])
    t1.record(compute)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    bm.close()
    return {"value": round(stats["kv"] / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "h2d_bytes_per_step": stats["h2d"] // ke, "d2h_bytes_per_step": stats["d2h"] // ke,
            "ms_per_step": round(ms / ke, 4), "steps": ke,
            "seq_steps_per_s": round(w.B * ke / (ms * 1e-3), 1),
            # host time per step outside its waits (allocator, planning, staging, launches)
            "host_busy_ms_per_step": round(1e3 * stats["host_s"] / ke, 4),
            "pipelining": "H2D of step i+1 on a copy stream and D2H of step i-1 on a result stream overlap the"
                          " kernels of step i; results read on the host two steps later"}


# ---------------------------------------------------------------------------
# Continuous-batching trace (the fifth workload, run step by step)
# ---------------------------------------------------------------------------

def run_trace(args, rank, world, local_rank):
    """Long-context trace: every step appends one token per running sequence
    (reshape_and_cache), decodes, frees finished sequences and admits seeded arrivals
    while the pool allows (their prompt K/V is written by one reshape_and_cache call,
    a synthetic prefill, outside the timed decode work).  Device time of the decode
    work (copy_blocks if any, reshape_and_cache, paged_attention_decode) is summed
    over the timed steps with CUDA events.

    The allocator's decisions depend on nothing the device computes, so they are made first, on
    the host, for every step (appends, copy-on-write pairs, tables, frees, admissions; their time
    is reported as allocator_us_per_step), and each step's tables, lengths, slots, pairs and
    inputs are staged on the device.  The timed pass then issues the device work in the serving
    loop's order with the host only launching, so the host stays ahead of the device and a slow
    host adds no idle time between a step's events.  Events are read after the last step; the
    oracle's sampled sequences are gathered on the device at their step and checked at the end."""
    import torch
    import paged_kv_cache_423_b200 as pkv

    device = bench_device(local_rank)
    torch.cuda.set_device(device)
    p = wl.TraceParams(steps=args.warmup + args.steps)
    initial, arrivals = wl.trace_events(p, seed=2000 + rank)
    rng = wl.rng_for(2001 + rank)
    order = rng.permutation(p.num_blocks).astype(np.int32)
    bm = pkv.BlockManager(p.num_blocks, p.block_size, order)
    g = torch.Generator(device=device)
    g.manual_seed(2002 + rank)
    shape = (p.num_blocks, p.num_kv_heads, p.block_size, p.head_dim)
    kc = torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    vc = torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    max_blocks = (p.len_hi + p.steps + p.block_size) // p.block_size + 1
    max_len = max_blocks * p.block_size
    ws = torch.empty(pkv.paged_attention_workspace_size(p.max_batch, p.num_heads, p.num_kv_heads, p.head_dim,
                                                        p.block_size, max_len), dtype=torch.uint8, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream()
    scale = wl.fp32_scale(p.head_dim)
    running = {}
    next_id = 0

    def up(a):
        """Host array -> device tensor without a host wait (pinned staging on a GPU)."""
        t = torch.from_numpy(np.ascontiguousarray(a))
        if device.type != "cuda":
            return t.to(device)
        return t.pin_memory().to(device, non_blocking=True)

    pending = []  # prompt writes of the sequences admitted since the last step: (slots, length)

    def admit(length, budget):
        nonlocal next_id
        if -(-length // p.block_size) > bm.num_free():
            return
        sid = next_id
        next_id += 1
        bm.add_seq(sid, length - 1)
        pending.append((up(bm.slots(sid, 0, length - 1)), length))
        running[sid] = budget

    # ---- pass 1, host only: the allocator's decisions for every step (appends, copy-on-write
    # pairs, tables, frees, admissions), each step's inputs staged on the device
    for length, budget in initial:
        admit(length, budget)
    alloc_s = 0.0  # host allocator time of the timed steps (append, export, frees)
    plan = []
    for step in range(p.steps):
        ids = sorted(running)
        rec = {"admits": pending[:], "n": len(ids)}
        pending.clear()
        if ids:
            a0 = time.perf_counter()
            slots, pairs = bm.append_slots(ids)
            tables, lens = bm.export_tables(ids, max_blocks)
            a_s = time.perf_counter() - a0
            rec.update(slots=up(slots), pairs=up(pairs) if len(pairs) else None, tables=up(tables), lens=up(lens),
                       tables_h=tables, lens_h=lens, ids=ids,
                       q=torch.randn((len(ids), p.num_heads, p.head_dim), generator=g, device=device).to(torch.bfloat16),
                       k=torch.randn((len(ids), p.num_kv_heads, p.head_dim), generator=g, device=device).to(torch.bfloat16),
                       ev=[torch.cuda.Event(enable_timing=True) for _ in range(4)])
            a0 = time.perf_counter()
            for sid in ids:
                running[sid] -= 1
                if running[sid] == 0:
                    bm.free_seq(sid)
                    del running[sid]
            if step >= args.warmup:
                alloc_s += a_s + time.perf_counter() - a0
        for length, budget in arrivals[step]:
            if len(running) < p.max_batch:
                admit(length, budget)
        plan.append(rec)
    torch.cuda.synchronize()

    seq_steps = 0
    kv_bytes = 0
    launches = 0
    timed = []  # the events of each timed step
    # CPU-baseline leg: the oracle on one sampled sequence of every 20th timed step, outside
    # the timed decode work; its output also checks the GPU's bf16 output for that sequence.
    oracle_leg = rank == 0 and not args.no_cpu_baseline
    ora = {"bytes": 0, "s": 0.0, "n": 0, "max_abs": 0.0, "error": None}
    ora_rng = wl.rng_for(2003)
    samples = []

    def oracle_sample_stash(ids, tables, lens, q, out):
        """Device copies of one sequence's query, output and blocks, taken in stream order
        after its step (the pool changes later)."""
        i = int(ora_rng.integers(len(ids)))
        L = int(lens[i])
        need = -(-L // p.block_size)
        blocks = up(tables[i][:need].astype(np.int64))
        samples.append((L, need, q[i:i + 1].clone(), out[i:i + 1].clone(), kc[blocks], vc[blocks]))

    def oracle_check(L, need, q1, out1, kb, vb):
        from threadpoolctl import threadpool_limits
        from oracle import paged_attention
        kh = kb.view(torch.int16).cpu().numpy().view(np.uint16)
        vh = vb.view(torch.int16).cpu().numpy().view(np.uint16)
        qh = q1.view(torch.int16).cpu().numpy().view(np.uint16)
        t0 = time.perf_counter()
        with threadpool_limits(limits=1):
            ref = paged_attention.paged_decode(qh, kh, vh, np.arange(need, dtype=np.int32)[None, :],
                                               np.array([L], np.int32), scale)
        ora["s"] += time.perf_counter() - t0
        ora["bytes"] += L * p.num_kv_heads * p.head_dim * 4
        ora["n"] += 1
        got = out1.float().cpu().numpy()
        ora["max_abs"] = max(ora["max_abs"], float(np.abs(got - ref).max()))

    # ---- pass 2: the device work in the order the serving loop issues it; the host only
    # launches, so it stays ahead of the device and no host time falls between a step's events
    out_all = torch.zeros((p.max_batch, p.num_heads, p.head_dim), dtype=torch.bfloat16, device=device)
    with ClockSampler(device) as clocks:
        for step, rec in enumerate(plan):
            for slots_d, length in rec["admits"]:  # synthetic prefill of the admitted prompts
                k = torch.randn((length - 1, p.num_kv_heads, p.head_dim), generator=g, device=device).to(torch.bfloat16)
                pkv.reshape_and_cache(k, k, kc, vc, slots_d, status=status)
            if rec["n"] == 0:
                continue
            ev, out = rec["ev"], out_all[:rec["n"]]
            ev[0].record(stream)
            if rec["pairs"] is not None:
                pkv.copy_blocks([kc], [vc], rec["pairs"], status=status)
            pkv.reshape_and_cache(rec["k"], rec["k"], kc, vc, rec["slots"], status=status)
            ev[1].record(stream)
            ev[2].record(stream)
            pkv.paged_attention_decode(out, rec["q"], kc, vc, rec["tables"], rec["lens"], max_len, scale, ws,
                                       status=status)
            ev[3].record(stream)
            if step >= args.warmup:
                timed.append(ev)
                seq_steps += rec["n"]
                kv_bytes += int(rec["lens_h"].astype(np.int64).sum()) * p.num_kv_heads * p.head_dim * 4
                launches += 3 + (1 if rec["pairs"] is not None else 0) + 1  # + the split merge
                if oracle_leg and (step - args.warmup) % 20 == 0:
                    oracle_sample_stash(rec["ids"], rec["tables_h"], rec["lens_h"], rec["q"], out)
        torch.cuda.synchronize()
    # the step's kernels: the cache write (and copies), then the decode call; the host's
    # marshalling of the decode call between the two is not device work
    t_ms = sum(ev[0].elapsed_time(ev[1]) + ev[2].elapsed_time(ev[3]) for ev in timed)
    span_ms = sum(ev[0].elapsed_time(ev[3]) for ev in timed)
    for smp in samples:
        if ora["error"] is None:
            try:
                oracle_check(*smp)
            except Exception as e:  # the trace figure stands without its baseline
                ora["error"] = f"{type(e).__name__}: {e}"
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item():#x}")
    bm.close()
    peak, peak_kind = measured_hbm_gbs()
    value = kv_bytes / (t_ms * 1e-3) / 1e9
    return {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(t_ms / max(1, args.steps), 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "long_trace_continuous", "max_batch": p.max_batch, "num_heads": p.num_heads,
                       "num_kv_heads": p.num_kv_heads, "head_dim": p.head_dim, "block_size": p.block_size,
                       "num_blocks": p.num_blocks, "admitted": next_id,
                       "initial_lengths": f"U{{{p.len_lo}..{p.len_hi}}}", "budgets": f"U{{{p.budget_lo}..{p.budget_hi}}}",
                       "arrivals": f"Bernoulli({p.arrival_p}) per free slot per step, lengths U{{{p.len_lo}..{p.len_hi}}}",
                       "timed": "copy_blocks + reshape_and_cache, and paged_attention_decode, per step (events"
                                " around each call; the allocator's decisions for all steps made and staged on the"
                                " device first, the timed pass only launching, so the host stays ahead of the device;"
                                " ms_per_step_span = first kernel start to last kernel end of a step)"},
            "ms_per_step_span": round(span_ms / max(1, args.steps), 4),
            "seq_steps_per_s": round(seq_steps / (t_ms * 1e-3), 1), "pct_hbm_peak": round(100 * value / peak, 2),
            # the same with the host allocator's time per step added (made before the timed pass here)
            "seq_steps_per_s_with_allocator": round(seq_steps / (t_ms * 1e-3 + alloc_s), 1),
            "allocator_us_per_step": round(1e6 * alloc_s / max(1, args.steps), 2),
            "gpu_launches": launches, "clocks": clocks.summary(),
            **({"cpu_baseline": ({"unavailable": ora["error"]} if ora["error"] or not ora["n"] else
                                 {"value": round(ora["bytes"] / ora["s"] / 1e9, 4), "unit": "GB/s", "cores": 1,
                                  "kind": "oracle",
                                  "sample": f"one sequence of every 20th timed step ({ora['n']} sequences, all "
                                            f"{p.num_heads} heads), float64 NumPy, 1 thread, {ora['s']:.1f} s",
                                  "max_abs_vs_gpu_bf16_out": round(ora["max_abs"], 5)})}
               if oracle_leg else {})}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline leg and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(w, step_inputs, n_seqs, rng):
    """Host copies of a sample of sequences (their blocks only) for the oracle."""
    import torch
    seqs = sorted(rng.choice(w.B, size=min(n_seqs, w.B), replace=False).tolist())
    lens = step_inputs["host_lens"] if "host_lens" in step_inputs else None
    tables = step_inputs["tables"].cpu().numpy()
    q = step_inputs["q"].view(torch.int16).cpu().numpy().view(np.uint16)
    items = []
    for s in seqs:
        need = -(-int(lens[s]) // w.bs)
        idx = torch.from_numpy(tables[s][:need].astype(np.int64)).to(w.device)
        kc = w.key_cache[idx].view(torch.int16).cpu().numpy().view(np.uint16)
        vc = w.value_cache[idx].view(torch.int16).cpu().numpy().view(np.uint16)
        items.append((q[s:s + 1], kc, vc, np.arange(need, dtype=np.int32)[None, :], lens[s:s + 1]))
    return items


def time_oracle(w, items, budget_s, repeat=False):
    """The decode oracle over the sampled sequences, 1 thread: one pass, stopped early once
    budget_s is spent, or (repeat) pass after pass until about budget_s of work; at least one
    sequence.  Returns bytes, seconds and sequences done."""
    from threadpoolctl import threadpool_limits
    from oracle import paged_attention
    done_bytes = 0
    t0 = time.perf_counter()
    n = 0
    with threadpool_limits(limits=1):
        while True:
            q, kc, vc, table, lens = items[n % len(items)]
            paged_attention.paged_decode(q, kc, vc, table, lens, w.scale)
            done_bytes += int(lens.sum()) * w.Hkv * w.D * 4
            n += 1
            if time.perf_counter() - t0 > budget_s or (not repeat and n == len(items)):
                break
    dt = time.perf_counter() - t0
    return done_bytes, dt, n


def _oracle_one(task):
    """One sequence through the oracle in a worker process (1 BLAS thread), its arrays
    memory-mapped from the sample directory; returns its tokens."""
    from threadpoolctl import threadpool_limits
    from oracle import paged_attention
    folder, i, scale = task
    q, kc, vc, table, lens = (np.load(os.path.join(folder, f"{i}_{k}.npy"), mmap_mode="r")
                              for k in ("q", "kc", "vc", "table", "lens"))
    with threadpool_limits(limits=1):
        paged_attention.paged_decode(q, kc, vc, table, lens, scale)
    return int(lens.sum())


def _noop(_):
    return 0


def time_oracle_all_cores(w, items):
    """The same sequences on every host core the process may use: a pool of spawned
    workers (spawn, not fork: the parent holds a CUDA context), started and warmed
    before the clock starts.  The sample is written once to a tmpfs folder that the
    workers memory-map (nothing is pickled), and it is processed `cores` times, one
    sequence per task, so the ideal time equals the 1-core time of one pass."""
    import multiprocessing as mp
    import shutil
    import tempfile
    cores = len(os.sched_getaffinity(0))
    need = sum(sum(np.asarray(x).nbytes for x in item) for item in items)
    shm = "/dev/shm"
    use_shm = os.path.isdir(shm) and shutil.disk_usage(shm).free > 2 * need + (64 << 20)
    folder = tempfile.mkdtemp(prefix="pkv_oracle_", dir=shm if use_shm else None)
    try:
        for i, (q, kc, vc, table, lens) in enumerate(items):
            for k, arr in (("q", q), ("kc", kc), ("vc", vc), ("table", table), ("lens", lens)):
                np.save(os.path.join(folder, f"{i}_{k}.npy"), np.ascontiguousarray(arr))
        work = [(folder, i, w.scale) for _ in range(cores) for i in range(len(items))]
        with mp.get_context("spawn").Pool(cores) as pool:
            pool.map(_noop, range(4 * cores), chunksize=1)
            t0 = time.perf_counter()
            toks = sum(pool.map(_oracle_one, work, chunksize=1))
            dt = time.perf_counter() - t0
    finally:
        shutil.rmtree(folder, ignore_errors=True)
    return toks * w.Hkv * w.D * 4, dt, cores


def cpu_baseline(w, step_inputs, budget_s=10.0):
    items = oracle_sample(w, step_inputs, 128, wl.rng_for(77))
    done, dt, n = time_oracle(w, items, budget_s, repeat=True)
    distinct = min(n, len(items))
    out = {"value": round(done / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": f"{n} sequence evaluations over {distinct} sampled sequences of the {w.label} batch "
                     f"(all {w.Hq} heads each, {n / len(items):.1f} passes), float64 NumPy, 1 thread, {dt:.1f} s"}
    try:
        done_all, dt_all, cores = time_oracle_all_cores(w, items[:distinct])
        out["all_cores"] = {"value": round(done_all / dt_all / 1e9, 4), "unit": "GB/s", "cores": cores,
                            "sample": f"the same {distinct} sequences, {cores} passes, over {cores} spawned worker "
                                      f"processes, {dt_all:.1f} s"}
    except Exception as e:  # the 1-core figure stands on its own
        out["all_cores"] = {"unavailable": f"{type(e).__name__}: {e}"}
    return out


def oracle_sample_fp8(w, step_inputs, n_seqs, rng):
    """Host copies of a sample of sequences of an 8-bit pool (their blocks only)."""
    import torch
    seqs = sorted(rng.choice(w.B, size=min(n_seqs, w.B), replace=False).tolist())
    lens = step_inputs["host_lens"]
    tables = step_inputs["tables"].cpu().numpy()
    q = step_inputs["q"].view(torch.int16).cpu().numpy().view(np.uint16)
    ks, vs = w.k_scale.cpu().numpy(), w.v_scale.cpu().numpy()
    items = []
    for s in seqs:
        need = -(-int(lens[s]) // w.bs)
        idx = torch.from_numpy(tables[s][:need].astype(np.int64)).to(w.device)
        items.append((q[s:s + 1], w.key_cache[idx].cpu().numpy(), w.value_cache[idx].cpu().numpy(), ks, vs,
                      np.arange(need, dtype=np.int32)[None, :], lens[s:s + 1]))
    return items


def time_oracle_fp8(w, items, budget_s, repeat=False):
    """The 8-bit decode oracle on sampled sequences, 1 thread, as time_oracle; KV bytes at
    1 B/value."""
    from threadpoolctl import threadpool_limits
    from oracle import fp8
    done = n = 0
    t0 = time.perf_counter()
    with threadpool_limits(limits=1):
        while True:
            q, kc, vc, ks, vs, table, lens = items[n % len(items)]
            fp8.paged_decode_fp8(q, kc, vc, ks, vs, table, lens, w.scale)
            done += int(lens.sum()) * w.Hkv * w.D * 2
            n += 1
            if time.perf_counter() - t0 > budget_s or (not repeat and n == len(items)):
                break
    return done, time.perf_counter() - t0, n


def cpu_baseline_fp8(w, step_inputs, budget_s=10.0):
    items = oracle_sample_fp8(w, step_inputs, 128, wl.rng_for(77))
    done, dt, n = time_oracle_fp8(w, items, budget_s, repeat=True)
    return {"value": round(done / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} sequence evaluations over {min(n, len(items))} sampled sequences of the {w.label} "
                      f"batch over the 8-bit pool (all {w.Hq} heads each, {n / len(items):.1f} passes), "
                      f"float64 NumPy, 1 thread, {dt:.1f} s"}


# ---------------------------------------------------------------------------
# Prefill / chunked prefill
# ---------------------------------------------------------------------------

def prefill_flops(query_lens, context_lens, num_heads, head_dim):
    """Algorithmic FLOPs of one prefill call: every query row of every head sees
    p + 1 keys (p its position); scores and the weighted sum cost 2 * D each per key."""
    visible = 0
    for n, L in zip(np.asarray(query_lens, np.int64), np.asarray(context_lens, np.int64)):
        visible += int(n) * (int(L) - int(n)) + int(n) * (int(n) + 1) // 2
    return 4 * head_dim * num_heads * visible


class PrefillWorkload:
    """One chunked-prefill batch resident on the device; per-step query/K/V states
    drawn on the host and uploaded before timing; the allocator gives tables and the
    chunk tokens' slots."""

    def __init__(self, name, n_states, seed, device, native=True):
        """native=False (the reference arm): the library is not loaded, the tables come
        from the allocator's reference model and no workspace is allocated."""
        import torch
        if native:
            import paged_kv_cache_423_b200 as pkv
        else:
            pkv = None
        self.pkv = pkv
        b = wl.make_prefill_batch(name, with_data=False)
        self.b = b
        self.name = name
        bm = (pkv.BlockManager if native else ModelManager)(b.num_blocks, b.block_size, b.free_order)
        ids = list(range(b.num_seqs))
        slots = []
        for s in ids:
            bm.add_seq(s, int(b.context_lens[s]))
            n = int(b.query_lens[s])
            slots.append(bm.slots(s, int(b.context_lens[s]) - n, n))
        tables, lens = bm.export_tables(ids, b.max_blocks)
        bm.close()
        self.slots = torch.from_numpy(np.concatenate(slots)).to(device)
        self.tables = torch.from_numpy(tables).to(device)
        self.lens = torch.from_numpy(lens).to(device)
        self.qstart = torch.from_numpy(b.query_start).to(device)
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        shape = (b.num_blocks, b.num_kv_heads, b.block_size, b.head_dim)
        self.key_cache = torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
        self.value_cache = torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
        rng = wl.rng_for(seed + 1)
        T = b.total_q
        self.host = []
        for _ in range(n_states):
            q = wl.bf16_normal(rng, (T, b.num_heads, b.head_dim))
            k, v = wl.new_tokens(rng, T, b.num_kv_heads, b.head_dim)
            self.host.append((q, k, v))
        self.ws = None if pkv is None else torch.empty(
            pkv.paged_attention_prefill_workspace_size(b.num_seqs, T, b.num_heads, b.num_kv_heads),
            dtype=torch.uint8, device=device)
        self.flops = prefill_flops(b.query_lens, b.context_lens, b.num_heads, b.head_dim)

    def step(self, q, k, v, out, status, ev=None, stream=None):
        b = self.b
        self.pkv.reshape_and_cache(k, v, self.key_cache, self.value_cache, self.slots, status=status)
        if ev is not None:
            ev[0].record(stream)
        self.pkv.paged_attention_prefill(out, q, self.key_cache, self.value_cache, self.tables, self.qstart, self.lens,
                                         b.max_context_len, b.scale, self.ws, status=status)
        if ev is not None:
            ev[1].record(stream)


def prefill_oracle_rate(pw, q_bits, budget_s, rng):
    """FLOPs done and seconds spent by the float64 prefill oracle on randomly sampled
    query rows (1 thread).  Only the oracle call is timed; fetching the row's pages
    from the device is not.  Runs until about `budget_s` seconds have passed."""
    import torch
    from threadpoolctl import threadpool_limits
    from oracle import prefill
    b = pw.b
    tables = pw.tables.cpu().numpy()
    done, work_t, n = 0, 0.0, 0
    wall0 = time.perf_counter()
    with threadpool_limits(limits=1):
        while n == 0 or time.perf_counter() - wall0 < budget_s:
            s = int(rng.integers(b.num_seqs))
            nq = int(b.query_lens[s])
            if nq == 0:
                continue
            i = int(rng.integers(nq))
            pos = int(b.context_lens[s]) - nq + i
            need = pos // b.block_size + 1
            idx = torch.from_numpy(tables[s][:need].astype(np.int64)).to(pw.key_cache.device)
            kc = pw.key_cache[idx].view(torch.int16).cpu().numpy().view(np.uint16)
            vc = pw.value_cache[idx].view(torch.int16).cpu().numpy().view(np.uint16)
            row = int(b.query_start[s]) + i
            tq = time.perf_counter()
            prefill.prefill_rows(q_bits[row:row + 1], kc, vc, np.arange(need, dtype=np.int32)[None, :],
                                 np.array([0, 1], np.int32), np.array([pos + 1], np.int32), b.scale, [0])
            work_t += time.perf_counter() - tq
            done += 4 * b.head_dim * b.num_heads * (pos + 1)
            n += 1
    return done, work_t, n


def run_prefill(args, rank, world, local_rank):
    import torch
    device = bench_device(local_rank)
    torch.cuda.set_device(device)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=device)
    n_states = 2
    pw = PrefillWorkload(args.workload, n_states, seed=2000 + rank, device=device)
    b = pw.b
    dev_states = [(to_dev(q, device), to_dev(k, device), to_dev(v, device)) for q, k, v in pw.host]
    out = torch.empty((b.total_q, b.num_heads, b.head_dim), dtype=torch.bfloat16, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        pw.step(*dev_states[i % n_states], out, status)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(device) as clocks:
        t0.record(stream)
        for j in range(args.steps):
            pw.step(*dev_states[j % n_states], out, status, ev[j], stream)
        t1.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item():#x}")
    ms = t0.elapsed_time(t1)
    k_ms = sum(a.elapsed_time(c) for a, c in ev)
    ms_max, flops_all = aggregate_over_ranks(ms, pw.flops * args.steps, dist, device)
    value = flops_all / (ms_max * 1e-3) / 1e12
    peak, peak_kind = measured_bf16_tflops()
    achieved = pw.flops * args.steps / (k_ms * 1e-3) / 1e12

    # e2e: q, chunk K/V from pinned host memory, output back to pinned memory, every step
    ke = max(1, min(args.steps, args.e2e_steps))
    host_in = [tuple(torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()
                     for a in st) for st in pw.host]
    out_host = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * 2 for t in host_in[0])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for j in range(ke):
        hq, hk, hv = host_in[j % n_states]
        dq, dk, dv = dev_states[j % n_states]
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        pw.step(dq, dk, dv, out, status)
        out_host.copy_(out, non_blocking=True)
        stream.synchronize()
        _ = float(out_host[0, 0, 0])
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = e0.elapsed_time(e1)
    result = {
        "metric": METRIC_PREFILL, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": b.name, "num_seqs": b.num_seqs, "num_heads": b.num_heads,
                   "num_kv_heads": b.num_kv_heads, "head_dim": b.head_dim, "block_size": b.block_size,
                   "query_tokens": b.total_q, "query_lens": b.query_lens.tolist(),
                   "context_lens": b.context_lens.tolist(), "flops_per_step": pw.flops,
                   "l2": "K/V of the batch (>= 0.6 GB) larger than L2; no flush",
                   "parallelism": f"replicas{world}" if world > 1 else "single"},
        "pct_tensor_peak": round(100 * value / world / peak, 2),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": recorded_traffic(b.name, "prefill", pw.flops),
                     "algorithmic_flops_per_launch": pw.flops, "peak_kind": peak_kind,
                     "kernel": "paged_attention_prefill: plan + tcgen05 kernel",
                     "ms_per_launch": round(k_ms / args.steps, 4)},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks.summary(),
        "e2e": {"value": round(pw.flops * ke / (e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": out_host.numel() * 2,
                "ms_per_step": round(e_ms / ke, 4), "steps": ke, "pipelining": "none (copy, compute, copy back, sync)"},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        done, dt, n = prefill_oracle_rate(pw, pw.host[0][0], args.cpu_budget, wl.rng_for(79))
        result["cpu_baseline"] = {"value": round(done / dt / 1e12, 6), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                                  "sample": f"{n} random query rows of the {b.name} batch (all {b.num_heads} heads), "
                                            f"float64 NumPy oracle, 1 thread, {dt:.1f} s"}
    if dist:
        dist.destroy_process_group()
    return result


# ---------------------------------------------------------------------------
# Swap (device <-> pinned host)
# ---------------------------------------------------------------------------

SWAP_SHAPE = (40, 16, 128)      # LLaMA-13B: 40 kv heads x 16 tokens x 128 (bf16): 160 KiB per K or V block
SWAP_PAIRS = 256


def run_swap(args, rank, world, local_rank):
    import torch
    import paged_kv_cache_423_b200 as pkv
    device = bench_device(local_rank)
    torch.cuda.set_device(device)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=device)
    NB, HB = 4096, 1024
    g = torch.Generator(device=device)
    g.manual_seed(3000 + rank)
    dk = torch.randn((NB,) + SWAP_SHAPE, generator=g, device=device).to(torch.bfloat16)
    dv = torch.randn((NB,) + SWAP_SHAPE, generator=g, device=device).to(torch.bfloat16)
    hk = torch.empty((HB,) + SWAP_SHAPE, dtype=torch.bfloat16).pin_memory()
    hv = torch.empty((HB,) + SWAP_SHAPE, dtype=torch.bfloat16).pin_memory()
    rng = wl.rng_for(3100 + rank)
    plans = []
    for _ in range(8):
        src = rng.permutation(NB)[:SWAP_PAIRS]
        dst = rng.permutation(HB)[:SWAP_PAIRS]
        back = rng.permutation(NB)[:SWAP_PAIRS]
        plans.append((torch.from_numpy(np.stack([src, dst], 1).astype(np.int64)).to(device),
                      torch.from_numpy(np.stack([dst, back], 1).astype(np.int64)).to(device)))
    status = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream()
    block_bytes = int(np.prod(SWAP_SHAPE)) * 2
    step_bytes = 4 * SWAP_PAIRS * block_bytes          # out and in, K and V

    def step(j):
        out_pairs, in_pairs = plans[j % len(plans)]
        pkv.swap_blocks(dk, hk, out_pairs, status=status)
        pkv.swap_blocks(dv, hv, out_pairs, status=status)
        pkv.swap_blocks(hk, dk, in_pairs, status=status)
        pkv.swap_blocks(hv, dv, in_pairs, status=status)

    for j in range(args.warmup):
        step(j)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    with ClockSampler(device) as clocks:
        t0.record(stream)
        for j in range(args.steps):
            step(j)
        t1.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item():#x}")
    ms = t0.elapsed_time(t1)
    ms_max, bytes_all = aggregate_over_ranks(ms, step_bytes * args.steps, dist, device)
    value = bytes_all / (ms_max * 1e-3) / 1e9
    # the link's own copy bandwidth: one pinned cudaMemcpyAsync each way of the same bytes per step
    big_d = torch.empty(step_bytes // 2, dtype=torch.uint8, device=device)
    big_h = torch.empty(step_bytes // 2, dtype=torch.uint8).pin_memory()
    m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(3):
        big_h.copy_(big_d, non_blocking=True)
        big_d.copy_(big_h, non_blocking=True)
    torch.cuda.synchronize()
    m0.record(stream)
    for _ in range(args.steps):
        big_h.copy_(big_d, non_blocking=True)
        big_d.copy_(big_h, non_blocking=True)
    m1.record(stream)
    torch.cuda.synchronize()
    link = step_bytes * args.steps / (m0.elapsed_time(m1) * 1e-3) / 1e9
    result = {
        "metric": METRIC_SWAP, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bytes", "data": "synthetic",
        "config": {"workload": SWAP_WORKLOAD, "block_shape": list(SWAP_SHAPE), "block_bytes": block_bytes,
                   "pairs_per_direction": SWAP_PAIRS, "bytes_per_step": step_bytes,
                   "parallelism": f"replicas{world}" if world > 1 else "single"},
        "roofline": {"bound": "host link", "achieved": round(value / world, 2), "peak": round(link, 2), "unit": "GB/s",
                     "frac": round(value / world / link, 4), "traffic": None,
                     "peak_kind": "measured in this run: pinned cudaMemcpyAsync D2H + H2D of the same bytes",
                     "kernel": "swap_blocks (4 launches per step)"},
        "gpu_launches": 4 * args.steps,
        "clocks": clocks.summary(),
        "e2e": {"value": round(value, 2), "unit": "GB/s", "h2d_bytes_per_step": step_bytes // 2,
                "d2h_bytes_per_step": step_bytes // 2,
                "note": "the timed step is itself a host<->device transfer of pinned memory"},
    }
    if dist:
        dist.destroy_process_group()
    return result


def run_reference(args, rank, world, local_rank):
    """The CPU oracle as the reference arm, on a bounded sample of the same workload."""
    import torch
    if rank != 0:
        return None
    device = bench_device(local_rank) if torch.cuda.is_available() else None
    if device is None:
        return {"impl": "reference", "unavailable": "no CUDA device to hold the synthetic workload"}
    torch.cuda.set_device(device)
    if args.workload in wl.PREFILL_WORKLOADS:
        return run_reference_prefill(args, world, device)
    if args.workload == SWAP_WORKLOAD:
        return run_reference_swap(args, world)
    kv8 = args.kv == "fp8"
    w = Workload(args.workload, 2, seed=1000, device=device, kv8=kv8, beams=args.beams, native=False)
    bm = w.new_manager()
    ids = w.seq_ids
    bm.append_slots(ids)
    tables, lens = bm.export_tables(ids, w.max_blocks)
    q, _, _ = w.host_step_inputs()
    st = {"tables": torch.from_numpy(tables), "host_lens": lens, "q": to_dev(q, device)}
    rng = wl.rng_for(78)
    sample_fn, timer = (oracle_sample_fp8, time_oracle_fp8) if kv8 else (oracle_sample, time_oracle)
    # size each step's sample so the whole run stays near --ref-budget seconds
    probe = sample_fn(w, st, 2, rng)
    _, dt_probe, n_probe = timer(w, probe, 1e9)
    per_seq = dt_probe / max(n_probe, 1)
    per_step = int(max(1, min(64, args.ref_budget / max(per_seq, 1e-6) / (args.warmup + args.steps))))
    for _ in range(args.warmup):
        timer(w, sample_fn(w, st, per_step, rng), 1e9)
    kv = 0
    dt_total = 0.0
    for _ in range(args.steps):
        b, dt, _n = timer(w, sample_fn(w, st, per_step, rng), 1e9)
        kv += b
        dt_total += dt
    value = kv / dt_total / 1e9
    sample = (f"{per_step} random sequences of the {w.label} batch per step (all {w.Hq} heads"
              f"{', 8-bit pool' if kv8 else ''}), float64 NumPy oracle, 1 thread")
    return {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * dt_total / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.label, "kv_dtype": args.kv, "num_seqs": w.B, "beams": w.beams,
                       "num_heads": w.Hq, "num_kv_heads": w.Hkv, "head_dim": w.D, "block_size": w.bs},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference_prefill(args, world, device):
    pw = PrefillWorkload(args.workload, 1, seed=2000, device=device, native=False)
    rng = wl.rng_for(80)
    per_step = max(0.05, args.ref_budget / (args.warmup + args.steps))
    for _ in range(args.warmup):
        prefill_oracle_rate(pw, pw.host[0][0], per_step, rng)
    done = dt = 0.0
    for _ in range(args.steps):
        d, t, _n = prefill_oracle_rate(pw, pw.host[0][0], per_step, rng)
        done += d
        dt += t
    value = done / dt / 1e12
    b = pw.b
    sample = f"random query rows of the {b.name} batch (all {b.num_heads} heads), {per_step:.2f} s per step, " \
             "float64 NumPy oracle, 1 thread"
    return {"metric": METRIC_PREFILL, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * dt / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": b.name, "num_seqs": b.num_seqs, "num_heads": b.num_heads,
                       "num_kv_heads": b.num_kv_heads, "head_dim": b.head_dim, "block_size": b.block_size},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference_swap(args, world):
    from oracle import cache_ops
    rng = wl.rng_for(81)
    src = np.zeros((512,) + SWAP_SHAPE, np.uint16)
    dst = np.zeros((256,) + SWAP_SHAPE, np.uint16)
    block_bytes = int(np.prod(SWAP_SHAPE)) * 2
    pairs_n = 64
    for _ in range(args.warmup):
        cache_ops.swap_blocks(src, dst, np.stack([rng.permutation(512)[:pairs_n], rng.permutation(256)[:pairs_n]], 1))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        cache_ops.swap_blocks(src, dst, np.stack([rng.permutation(512)[:pairs_n], rng.permutation(256)[:pairs_n]], 1))
    dt = time.perf_counter() - t0
    # the oracle copies the whole destination pool once per call plus the pairs; count the pairs' bytes
    value = args.steps * pairs_n * block_bytes / dt / 1e9
    sample = f"{pairs_n} 13B-shaped blocks per step between two host arrays (NumPy), 1 thread"
    return {"metric": METRIC_SWAP, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * dt / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bytes", "data": "synthetic",
            "config": {"workload": SWAP_WORKLOAD, "block_shape": list(SWAP_SHAPE)}, "impl": "reference",
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--states", type=int, default=16, help="distinct precomputed decode steps replayed in turn")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama13b_mixed_bs16",
                    choices=sorted(wl.WORKLOADS) + sorted(wl.PREFILL_WORKLOADS) + [SWAP_WORKLOAD])
    ap.add_argument("--kv", choices=["bf16", "fp8"], default="bf16", help="element type of the decode pool")
    ap.add_argument("--path", choices=["auto", "simt", "tensor"], default="auto")
    ap.add_argument("--beams", type=int, default=1,
                    help="prefix_beams only: fork every sequence into this many beams before the first step")
    ap.add_argument("--shared", choices=["auto", "on", "off"], default="auto",
                    help="shared-prefix decode (blocks that adjacent rows share read once per kv head): auto = on "
                         "for the shared-prompt workload over a bf16 pool")
    ap.add_argument("--min-rows", type=int, default=None,
                    help="fewest rows a shared segment serves in the shared-prefix decode's plan"
                         " (default 2 over bf16 pools, 5 over 8-bit pools)")
    ap.add_argument("--key-chunk", type=int, default=0,
                    help="keys per part of a shared segment in the shared-prefix decode's plan (0 = automatic)")
    ap.add_argument("--trace", action="store_true",
                    help="run the long-context continuous-batching trace step by step (the fifth workload)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--ref-budget", type=float, default=60.0, help="seconds of oracle work in --impl reference")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.beams < 1 or (args.beams > 1 and (args.workload != "prefix_beams" or args.trace)):
        raise SystemExit("--beams N > 1 applies to --workload prefix_beams only")
    rank, world, local_rank = rank_info()
    if args.impl == "reference":
        res = run_reference(args, rank, world, local_rank)
    elif args.trace:
        res = run_trace(args, rank, world, local_rank)
    elif args.workload in wl.PREFILL_WORKLOADS:
        res = run_prefill(args, rank, world, local_rank)
    elif args.workload == SWAP_WORKLOAD:
        res = run_swap(args, rank, world, local_rank)
    else:
        res = run_ours(args, rank, world, local_rank)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
