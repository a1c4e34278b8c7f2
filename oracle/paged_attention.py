"""Oracle: single-token decode attention over a paged KV cache (float64, NumPy).

TEST INFRASTRUCTURE ONLY -- see the package docstring.

What it follows
  * intelliparadigm article "PagedAttention：操作系统分页思想的跨界创新", §2.1 核心设计原理,
    the paged_attention pseudo-code: the logical block of a position is
    position // block_size, the block table maps it to a physical page, K and V are
    loaded from those pages, and the result is softmax(query @ keys.T) @ values.
  * vLLM 初探 §1.4 (block-table figure): logical Block i -> a physical block anywhere
    in one shared pool; Outcome School explainer, "vLLM的核心创新：PagedAttention":
    fixed-size blocks (16 tokens) and a per-request block table that keeps the order.

Readings where the pages are silent (each listed in the design notes):
  * the scores are multiplied by the caller's ``scale`` (the pseudo-code has none);
  * the context of sequence s is tokens 0 .. L_s-1, the current token included;
  * grouped-query attention maps query head h to KV head h // (Hq / Hkv);
  * a sequence with L_s = 0 yields a zero output row.

Parity status: pinned (closed forms, a library attention routine, invariants).
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly (bf16 is the top half of fp32)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def gather_sequence(cache_bits: np.ndarray, table_row: np.ndarray, context_len: int) -> np.ndarray:
    """Contiguous float64 copy of one sequence's K (or V): [L, Hkv, D].

    Token t sits in logical block t // bs at row t % bs; the table row maps the
    logical block to its physical block (the pseudo-code's block_id and
    physical_page).  cache layout: [num_blocks, Hkv, bs, D]."""
    block_size = cache_bits.shape[2]
    positions = np.arange(context_len)
    physical = np.asarray(table_row)[positions // block_size]
    rows = positions % block_size
    # cache[physical[t], :, rows[t], :] for every t -> [L, Hkv, D]
    return bf16_bits_to_f64(cache_bits[physical, :, rows, :])


def attend(q: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float) -> np.ndarray:
    """Textbook softmax attention of one query vector over L keys/values (float64).

    q [D], keys [L, D], values [L, D] -> [D]."""
    z = float(scale) * (keys @ q)
    w = np.exp(z - z.max())
    w = w / w.sum()
    return w @ values


def paged_decode(query_bits, key_cache_bits, value_cache_bits, block_tables, context_lens, scale):
    """Decode attention for every (sequence, query head): float64 [B, Hq, D].

    query_bits [B, Hq, D] uint16; caches [NB, Hkv, bs, D] uint16; block_tables
    [B, max_blocks] int32; context_lens [B]; scale: the float32 value the caller
    passes to the GPU (used here widened to float64)."""
    num_seqs, num_heads, head_dim = query_bits.shape
    num_kv_heads = key_cache_bits.shape[1]
    group = num_heads // num_kv_heads
    scale64 = float(np.float32(scale))
    q_all = bf16_bits_to_f64(query_bits)
    out = np.zeros((num_seqs, num_heads, head_dim), dtype=np.float64)
    for s in range(num_seqs):
        length = int(context_lens[s])
        if length == 0:
            continue
        keys = gather_sequence(key_cache_bits, block_tables[s], length)
        values = gather_sequence(value_cache_bits, block_tables[s], length)
        for h in range(num_heads):
            kv_head = h // group
            out[s, h] = attend(q_all[s, h], keys[:, kv_head, :], values[:, kv_head, :], scale64)
    return out


def contiguous_decode(query_bits, keys_bits, values_bits, context_lens, scale):
    """Attention over the traditional contiguous layout (vLLM 初探 §1.4: one
    [heads, seq_len, head_dim] slab per request, pre-reserved to a maximum length).

    keys_bits / values_bits: [B, Hkv, max_len, D] uint16; only the first L_s rows count."""
    num_seqs, num_heads, _ = query_bits.shape
    num_kv_heads = keys_bits.shape[1]
    group = num_heads // num_kv_heads
    scale64 = float(np.float32(scale))
    q_all = bf16_bits_to_f64(query_bits)
    out = np.zeros(query_bits.shape, dtype=np.float64)
    for s in range(num_seqs):
        length = int(context_lens[s])
        if length == 0:
            continue
        for h in range(num_heads):
            kv_head = h // group
            keys = bf16_bits_to_f64(keys_bits[s, kv_head, :length])
            values = bf16_bits_to_f64(values_bits[s, kv_head, :length])
            out[s, h] = attend(q_all[s, h], keys, values, scale64)
    return out

