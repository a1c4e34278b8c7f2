"""Oracle: the two cache-writing operations of the decode step (bit copies).

TEST INFRASTRUCTURE ONLY -- see the package docstring.

reshape_and_cache
  Each new token's K and V go into the pool at its slot (Outcome School explainer,
  "LLM serving的基本流程与KV缓存": every decoded token adds one K/V pair that stays
  resident until the request ends).  slot = physical_block * block_size + row; the
  caller derives it from the block table.  A negative slot means "skip this row".
copy_blocks
  Copy-on-write of shared blocks (Outcome School explainer, "内存共享": beams share
  blocks until they diverge): for every (src, dst) pair, dst <- src in every layer,
  K and V.  All reads happen before any write (pairs are applied as one parallel copy).
swap_blocks
  The pool's overflow path (intelliparadigm article, §4.2 OOM错误: swap_space extends
  the cache into host memory): for every (src, dst) pair, block dst of the destination
  pool (host or device) <- block src of the source pool, K and V alike.  The two pools
  are different memories, so no pair can read what another writes.

Parity status: pinned (explicit element loops on tiny inputs, invariants).
"""
from __future__ import annotations

import numpy as np


def reshape_and_cache(key_bits, value_bits, key_cache_bits, value_cache_bits, slot_mapping):
    """Return new (key_cache, value_cache) with token t written at slot_mapping[t].

    key_bits / value_bits [T, Hkv, D] uint16; caches [NB, Hkv, bs, D] uint16."""
    block_size = key_cache_bits.shape[2]
    kc = key_cache_bits.copy()
    vc = value_cache_bits.copy()
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64)):
        if slot < 0:
            continue
        block, row = divmod(int(slot), block_size)
        kc[block, :, row, :] = key_bits[t]
        vc[block, :, row, :] = value_bits[t]
    return kc, vc


def copy_blocks(key_caches, value_caches, block_mapping):
    """Return new lists of caches with every pair's dst block replaced by its src block."""
    pairs = np.asarray(block_mapping, dtype=np.int64).reshape(-1, 2)
    out_k, out_v = [], []
    for kc, vc in zip(key_caches, value_caches):
        new_k, new_v = kc.copy(), vc.copy()
        for src, dst in pairs:
            new_k[dst] = kc[src]
            new_v[dst] = vc[src]
        out_k.append(new_k)
        out_v.append(new_v)
    return out_k, out_v


def swap_blocks(src_pool, dst_pool, block_mapping):
    """Return a new destination pool with dst_pool[dst] = src_pool[src] for every pair.

    Pools [NB, ...] of any element type (the two pools may differ in NB)."""
    pairs = np.asarray(block_mapping, dtype=np.int64).reshape(-1, 2)
    out = dst_pool.copy()
    for src, dst in pairs:
        out[dst] = src_pool[src]
    return out
