"""Seeded synthetic inputs for paged decode attention.

This module only draws inputs: context lengths, the placement of each sequence's
blocks in the shared physical pool, and bf16 data.  It holds none of the
attention, caching or allocation arithmetic, so both the CPU oracle (``oracle/``)
and the CUDA path (``paged_kv_cache_423_b200``) can take their inputs from it
without sharing any of the method's code.

Shapes follow the workloads the pages talk about: LLaMA-7B / 13B head shapes,
mixed 10-2000-token lengths (vLLM 初探 §1.1; intelliparadigm article §1),
a shared system prompt (vLLM 初探 §1.4; Outcome School explainer, "内存共享"),
and 5k+ contexts (intelliparadigm article §2.2 table, §4.2).  The pages name no
dataset or benchmark suite; these seeded draws stand in for the request mixes.

Layouts (all row-major, contiguous):
  query / key / value of new tokens : [T, H, D] bf16 (stored here as uint16 bits)
  key_cache / value_cache (one layer): [num_blocks, num_kv_heads, block_size, D] bf16
  block_tables                       : [B, max_blocks] int32, padded with 0
  context_lens                       : [B] int32
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

# Base seed and per-workload sub-seeds.
BASE_SEED = 0


def rng_for(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return uint16 bits.

    Inputs are finite normal draws, so no NaN handling is needed here."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_normal(rng: np.random.Generator, shape) -> np.ndarray:
    """N(0, 1) draws rounded to bf16, as uint16 bit patterns."""
    return f32_to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


@dataclasses.dataclass
class DecodeBatch:
    """One decode-attention call's worth of inputs (one layer)."""

    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    context_lens: np.ndarray        # [B] int32
    block_tables: np.ndarray        # [B, max_blocks] int32, pad 0
    scale: float                    # float32 value, e.g. 1/sqrt(D) rounded to fp32
    free_order: np.ndarray          # [NB] int32: seeded permutation of the pool
    seed: int
    query: np.ndarray | None = None         # [B, Hq, D] uint16 (bf16 bits)
    key_cache: np.ndarray | None = None     # [NB, Hkv, bs, D] uint16
    value_cache: np.ndarray | None = None   # [NB, Hkv, bs, D] uint16

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    def kv_bytes(self) -> int:
        """bf16 K+V bytes the valid tokens occupy (each (token, kv head) once)."""
        return int(self.context_lens.astype(np.int64).sum()) * self.num_kv_heads * self.head_dim * 2 * 2


def fp32_scale(head_dim: int) -> float:
    return float(np.float32(1.0 / math.sqrt(head_dim)))


def blocks_needed(lens: np.ndarray, block_size: int) -> np.ndarray:
    return (lens.astype(np.int64) + block_size - 1) // block_size


def place_blocks(lens: np.ndarray, block_size: int, free_order: np.ndarray,
                 shared_prefix_blocks: int = 0, max_blocks: int | None = None) -> np.ndarray:
    """Give each sequence its blocks by walking the seeded pool permutation in order.

    With ``shared_prefix_blocks = P``, the first P blocks taken go to every
    sequence's first P table entries (one shared system prompt); each sequence then
    takes its private blocks.  Returns the padded int32 table."""
    need = blocks_needed(lens, block_size)
    mb = int(need.max()) if len(lens) else 1
    if max_blocks is not None:
        mb = max(mb, max_blocks)
    tables = np.zeros((len(lens), max(mb, 1)), dtype=np.int32)
    cursor = 0
    prefix = free_order[cursor:cursor + shared_prefix_blocks]
    cursor += shared_prefix_blocks
    for s, n in enumerate(need):
        tables[s, :shared_prefix_blocks] = prefix
        private = int(n) - shared_prefix_blocks
        tables[s, shared_prefix_blocks:shared_prefix_blocks + private] = free_order[cursor:cursor + private]
        cursor += private
    if cursor > len(free_order):
        raise ValueError("pool too small for the drawn lengths")
    return tables


# ---------------------------------------------------------------------------
# Length distributions of the five workloads
# ---------------------------------------------------------------------------

def lens_tiny() -> np.ndarray:
    return np.array([1, 7, 16, 33], dtype=np.int32)


def lens_uniform(rng, n, lo, hi) -> np.ndarray:
    return rng.integers(lo, hi + 1, size=n).astype(np.int32)


def lens_mixed_13b(rng, n, short_mean=50, long_lo=1000, long_hi=2000, long_frac=0.3) -> np.ndarray:
    """70/30 mixture: geometric with mean ``short_mean`` (support >= 1) and U{long_lo..long_hi}."""
    is_long = rng.random(n) < long_frac
    short = rng.geometric(1.0 / short_mean, size=n)
    long = rng.integers(long_lo, long_hi + 1, size=n)
    return np.where(is_long, long, short).astype(np.int32)


WORKLOADS = {
    # name: (B, Hq, Hkv, D, bs)
    "tiny": (4, 2, 2, 64, 16),
    "llama7b": (64, 32, 32, 128, 16),
    "llama13b_mixed_bs16": (256, 40, 40, 128, 16),
    "llama13b_mixed_bs32": (256, 40, 40, 128, 32),
    "prefix_beams": (128, 32, 8, 128, 16),
    "long_trace": (16, 64, 8, 128, 32),
}

SUB_SEED = {name: i + 1 for i, name in enumerate(WORKLOADS)}

PREFIX_TOKENS = 1024  # shared system prompt of the prefix + beam workload


def draw_lengths(name: str, rng: np.random.Generator, num_seqs: int, length_scale: float = 1.0) -> np.ndarray:
    """Context lengths of ``name``; ``length_scale`` < 1 shrinks them for oracle-sized tests."""
    def sc(x):
        return max(1, int(round(x * length_scale)))

    if name == "tiny":
        return lens_tiny()[:num_seqs]
    if name == "llama7b":
        return lens_uniform(rng, num_seqs, sc(10), sc(2000))
    if name.startswith("llama13b_mixed"):
        return lens_mixed_13b(rng, num_seqs, short_mean=max(2, sc(50)), long_lo=sc(1000), long_hi=sc(2000))
    if name == "prefix_beams":
        suffix = lens_uniform(rng, num_seqs, sc(10), sc(500))
        return (sc(PREFIX_TOKENS) + suffix).astype(np.int32)
    if name == "long_trace":
        return lens_uniform(rng, num_seqs, sc(5000), sc(32000))
    raise KeyError(name)


def make_decode_batch(name: str, *, seed: int | None = None, num_seqs: int | None = None,
                      length_scale: float = 1.0, pool_factor: float = 1.2, extra_blocks: int = 0,
                      with_data: bool = True, num_heads: int | None = None,
                      num_kv_heads: int | None = None, head_dim: int | None = None,
                      block_size: int | None = None, lengths: np.ndarray | None = None,
                      max_blocks: int | None = None) -> DecodeBatch:
    """Draw one decode batch of workload ``name``.

    The pool holds ``ceil(pool_factor * sum(blocks needed)) + extra_blocks`` blocks
    (64 for the tiny workload); every block of it, used or not, is filled with
    N(0,1) bf16 data so stale rows past a context end hold real numbers.
    Smaller variants (fewer sequences, shorter lengths, other head counts) keep the
    same distributions and are used where the oracle has to finish in seconds."""
    B0, Hq0, Hkv0, D0, bs0 = WORKLOADS[name]
    B = B0 if num_seqs is None else num_seqs
    Hq = Hq0 if num_heads is None else num_heads
    Hkv = Hkv0 if num_kv_heads is None else num_kv_heads
    D = D0 if head_dim is None else head_dim
    bs = bs0 if block_size is None else block_size
    seed = BASE_SEED * 1000 + SUB_SEED[name] if seed is None else seed
    rng = rng_for(seed)
    lens = draw_lengths(name, rng, B, length_scale) if lengths is None else np.asarray(lengths, np.int32)
    B = len(lens)
    shared = 0
    if name == "prefix_beams":
        shared = max(1, int(round(PREFIX_TOKENS * length_scale))) // bs
    need = blocks_needed(lens, bs)
    if name == "tiny" and num_seqs is None and lengths is None:
        nb = 64
    else:
        used = int(need.sum()) - shared * max(B - 1, 0)
        nb = int(math.ceil(pool_factor * used)) + extra_blocks
        nb = max(nb, used, 1)
    free_order = rng.permutation(nb).astype(np.int32)
    tables = place_blocks(lens, bs, free_order, shared_prefix_blocks=shared, max_blocks=max_blocks)
    batch = DecodeBatch(name=name, num_seqs=B, num_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                        block_size=bs, num_blocks=nb, context_lens=lens, block_tables=tables,
                        scale=fp32_scale(D), free_order=free_order, seed=seed)
    if with_data:
        batch.query = bf16_normal(rng, (B, Hq, D))
        batch.key_cache = bf16_normal(rng, (nb, Hkv, bs, D))
        batch.value_cache = bf16_normal(rng, (nb, Hkv, bs, D))
    return batch


def new_tokens(rng: np.random.Generator, num_tokens: int, num_kv_heads: int, head_dim: int):
    """K and V of ``num_tokens`` new tokens, [T, Hkv, D] bf16 bits each."""
    return (bf16_normal(rng, (num_tokens, num_kv_heads, head_dim)),
            bf16_normal(rng, (num_tokens, num_kv_heads, head_dim)))


# ---------------------------------------------------------------------------
# Long-context continuous-batching trace (the fifth workload)
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class TraceParams:
    max_batch: int = 16
    num_heads: int = 64
    num_kv_heads: int = 8
    head_dim: int = 128
    block_size: int = 32
    len_lo: int = 5000
    len_hi: int = 32000
    budget_lo: int = 1
    budget_hi: int = 400
    steps: int = 200
    arrival_p: float = 0.5
    num_blocks: int = 19661  # ceil(1.2 * 16 * 32768 / 32)


def trace_events(params: TraceParams, seed: int):
    """Seeded request stream for the trace: initial requests and, per step, the
    per-free-slot arrival draws.  Returns (initial [(len, budget)], arrivals) where
    ``arrivals[step]`` is a list of (len, budget) offered at that step, one per
    potential free slot (the consumer admits them while the pool allows)."""
    rng = rng_for(seed)
    initial = [(int(rng.integers(params.len_lo, params.len_hi + 1)),
                int(rng.integers(params.budget_lo, params.budget_hi + 1))) for _ in range(params.max_batch)]
    arrivals = []
    for _ in range(params.steps):
        offers = []
        for _slot in range(params.max_batch):
            if rng.random() < params.arrival_p:
                offers.append((int(rng.integers(params.len_lo, params.len_hi + 1)),
                               int(rng.integers(params.budget_lo, params.budget_hi + 1))))
        arrivals.append(offers)
    return initial, arrivals


# ---------------------------------------------------------------------------
# Prefill / chunked-prefill batches
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class PrefillBatch:
    """One prefill-attention call's worth of inputs (one layer).

    Sequence s already holds context_lens[s] tokens in the pool, of which the last
    query_lens[s] are this call's new tokens (its chunk); their query rows are packed
    at query_start[s] .. query_start[s+1]-1."""

    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    query_lens: np.ndarray          # [B] int32
    context_lens: np.ndarray        # [B] int32 (earlier tokens + this chunk)
    query_start: np.ndarray         # [B+1] int32
    block_tables: np.ndarray        # [B, max_blocks] int32, pad 0
    scale: float
    free_order: np.ndarray
    seed: int
    query: np.ndarray | None = None         # [T, Hq, D] uint16
    key_cache: np.ndarray | None = None     # [NB, Hkv, bs, D] uint16
    value_cache: np.ndarray | None = None

    @property
    def total_q(self) -> int:
        return int(self.query_start[-1])

    @property
    def max_query_len(self) -> int:
        return int(self.query_lens.max()) if self.num_seqs else 0

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])


PREFILL_WORKLOADS = {
    # name: (B, Hq, Hkv, D, bs, chunk, earlier_lo, earlier_hi)
    # 8 chunks of 512 tokens = 4096 batched tokens (intelliparadigm article §4.1/§4.2:
    # chunked_prefill_token_size=512, max_num_batched_tokens=4096), LLaMA-13B heads.
    "chunked_prefill_13b": (8, 40, 40, 128, 16, 512, 0, 8192),
    # the same chunking on 10k+-token contexts (§4.2) with grouped-query heads
    "chunked_prefill_long_gqa": (8, 64, 8, 128, 32, 512, 4096, 28672),
}

PREFILL_SUB_SEED = {name: 100 + i for i, name in enumerate(PREFILL_WORKLOADS)}


def make_prefill_batch(name: str, *, seed: int | None = None, num_seqs: int | None = None,
                       length_scale: float = 1.0, with_data: bool = True, num_heads: int | None = None,
                       num_kv_heads: int | None = None, head_dim: int | None = None,
                       block_size: int | None = None, query_lens=None, earlier_lens=None,
                       pool_factor: float = 1.2) -> PrefillBatch:
    """Draw one prefill batch.  A quarter of the sequences (at least one when B > 1) end
    their prompt inside this call with a shorter, ragged chunk U{1..chunk}; the rest
    take a full chunk.  Earlier (already cached) lengths are U{lo..hi}, scaled by
    ``length_scale``.  Explicit ``query_lens`` / ``earlier_lens`` override the draws."""
    B0, Hq0, Hkv0, D0, bs0, chunk0, lo, hi = PREFILL_WORKLOADS[name]
    B = B0 if num_seqs is None else num_seqs
    Hq = Hq0 if num_heads is None else num_heads
    Hkv = Hkv0 if num_kv_heads is None else num_kv_heads
    D = D0 if head_dim is None else head_dim
    bs = bs0 if block_size is None else block_size
    seed = BASE_SEED * 1000 + PREFILL_SUB_SEED[name] if seed is None else seed
    rng = rng_for(seed)
    chunk = max(1, int(round(chunk0 * length_scale)))
    if query_lens is None:
        qlens = np.full(B, chunk, dtype=np.int32)
        ragged = rng.random(B) < 0.25
        if B > 1 and not ragged.any():
            ragged[rng.integers(B)] = True
        qlens[ragged] = rng.integers(1, chunk + 1, size=int(ragged.sum()))
    else:
        qlens = np.asarray(query_lens, np.int32)
    B = len(qlens)
    if earlier_lens is None:
        earlier = rng.integers(int(round(lo * length_scale)), int(round(hi * length_scale)) + 1, size=B)
    else:
        earlier = np.asarray(earlier_lens)
    lens = (earlier + qlens).astype(np.int32)
    qstart = np.zeros(B + 1, dtype=np.int32)
    qstart[1:] = np.cumsum(qlens)
    need = blocks_needed(lens, bs)
    nb = max(int(math.ceil(pool_factor * int(need.sum()))), 1)
    free_order = rng.permutation(nb).astype(np.int32)
    tables = place_blocks(lens, bs, free_order)
    batch = PrefillBatch(name=name, num_seqs=B, num_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=bs,
                         num_blocks=nb, query_lens=qlens, context_lens=lens, query_start=qstart,
                         block_tables=tables, scale=fp32_scale(D), free_order=free_order, seed=seed)
    if with_data:
        batch.query = bf16_normal(rng, (int(qstart[-1]), Hq, D))
        batch.key_cache = bf16_normal(rng, (nb, Hkv, bs, D))
        batch.value_cache = bf16_normal(rng, (nb, Hkv, bs, D))
    return batch


def kv_scales(rng: np.random.Generator, num_kv_heads: int, lo: float = 1.0 / 64, hi: float = 1.0 / 32) -> np.ndarray:
    """Seeded per-kv-head float32 scales of an 8-bit cache: N(0,1) data divided by a
    scale in [1/64, 1/32] spans about +-320 before saturation at 448."""
    return rng.uniform(lo, hi, size=num_kv_heads).astype(np.float32)


def e4m3_codes(rng: np.random.Generator, shape) -> np.ndarray:
    """Seeded 8-bit (e4m3) pool contents drawn directly as bit patterns: random sign,
    exponent field around 8 (values of magnitude ~1..4 before the scale), uniform
    mantissa, never the NaN pattern.  Pure integer draws, no rounding arithmetic."""
    sign = rng.integers(0, 2, size=shape)
    exp = np.clip(np.rint(rng.normal(8.0, 1.5, size=shape)), 0, 15).astype(np.int64)
    mant = rng.integers(0, 8, size=shape)
    mant = np.where((exp == 15) & (mant == 7), 6, mant)
    return ((sign << 7) | (exp << 3) | mant).astype(np.uint8)
