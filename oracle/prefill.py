"""Oracle: prefill and chunked-prefill attention over a paged KV cache (float64, NumPy).

TEST INFRASTRUCTURE ONLY -- see the package docstring.

What it follows
  * Outcome School explainer, "LLM serving的基本流程与KV缓存": in the prefill phase the
    model reads the whole prompt at once and computes and stores the K/V of every
    prompt token; decode then needs the K/V of all earlier tokens.
  * intelliparadigm article, §4.1 (批处理策略调优) and §4.2 (长序列性能下降): chunked
    prefill splits a long prompt into pieces (e.g. 512 tokens) that are processed
    batch by batch.
  * intelliparadigm article, §2.1: attention reads K/V page by page through the block
    table (the same gather as decode).

Readings where the pages are silent (each listed in the design notes):
  * A sequence's new tokens (its chunk) are the last n_s of its L_s cached tokens;
    their K/V are already in the pool when attention runs.  Chunk row i is the token
    at position p = L_s - n_s + i and attends to positions 0 .. p (causal: a token
    sees itself and everything before it, never a later token).
  * The query rows of all sequences are packed one after another; sequence s owns
    rows query_start[s] .. query_start[s+1]-1.
  * Scale, grouped-query head mapping and bf16 inputs as in decode.

Parity status: pinned (library causal attention, reduction to decode, chunking
invariance, closed forms).
"""
from __future__ import annotations

import numpy as np

from .paged_attention import attend, bf16_bits_to_f64, gather_sequence


def paged_prefill(query_bits, key_cache_bits, value_cache_bits, block_tables, query_start, context_lens, scale):
    """Causal attention of every new query row over its sequence's paged K/V.

    query_bits [T, Hq, D] uint16 (T = query_start[-1]); caches [NB, Hkv, bs, D]
    uint16; block_tables [B, max_blocks]; query_start [B+1]; context_lens [B].
    Returns float64 [T, Hq, D]."""
    total, num_heads, head_dim = query_bits.shape
    num_kv_heads = key_cache_bits.shape[1]
    group = num_heads // num_kv_heads
    scale64 = float(np.float32(scale))
    q_all = bf16_bits_to_f64(query_bits)
    out = np.zeros((total, num_heads, head_dim), dtype=np.float64)
    starts = [int(x) for x in query_start]
    for s in range(len(starts) - 1):
        n = starts[s + 1] - starts[s]
        length = int(context_lens[s])
        if n == 0:
            continue
        keys = gather_sequence(key_cache_bits, block_tables[s], length)
        values = gather_sequence(value_cache_bits, block_tables[s], length)
        for i in range(n):
            position = length - n + i
            row = starts[s] + i
            for h in range(num_heads):
                kv_head = h // group
                out[row, h] = attend(q_all[row, h], keys[:position + 1, kv_head, :],
                                     values[:position + 1, kv_head, :], scale64)
    return out


def prefill_rows(query_bits, key_cache_bits, value_cache_bits, block_tables, query_start, context_lens, scale,
                 rows):
    """The same definition for selected packed rows only: float64 [len(rows), Hq, D].

    Used to check sampled rows of full-size batches."""
    starts = np.asarray(query_start, dtype=np.int64)
    num_heads = query_bits.shape[1]
    num_kv_heads = key_cache_bits.shape[1]
    group = num_heads // num_kv_heads
    scale64 = float(np.float32(scale))
    out = np.zeros((len(rows), num_heads, query_bits.shape[2]), dtype=np.float64)
    for j, row in enumerate(rows):
        s = int(np.searchsorted(starts, row, side="right")) - 1
        n = int(starts[s + 1] - starts[s])
        length = int(context_lens[s])
        position = length - n + (int(row) - int(starts[s]))
        keys = gather_sequence(key_cache_bits, block_tables[s], position + 1)
        values = gather_sequence(value_cache_bits, block_tables[s], position + 1)
        q = bf16_bits_to_f64(query_bits[row])
        for h in range(num_heads):
            out[j, h] = attend(q[h], keys[:, h // group, :], values[:, h // group, :], scale64)
    return out

