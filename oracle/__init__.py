"""CPU oracle for the paged KV-cache decode path -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct restatements of what the path computes, in float64
NumPy (attention) and plain Python (cache ops, allocator).  They share no code
with the CUDA library and import nothing from it.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference legs may
import or call anything here; the product path never does.

Modules
  paged_attention  decode attention through block tables (gather + textbook softmax)
  prefill          prefill / chunked-prefill attention (causal, multi-token queries)
  fp8              e4m3 codec, the quantising cache write, decode over an 8-bit pool
  cache_ops        reshape_and_cache (slot scatter), copy_blocks (copy-on-write copy),
                   swap_blocks (device <-> host pool copy)
  block_manager    reference model of the block allocator and per-sequence tables,
                   with swap space and automatic prefix caching

Every function is pinned by ``tests/test_oracle_pins.py``,
``tests/test_oracle_prefill_pins.py``, ``tests/test_oracle_fp8_pins.py`` and
``tests/test_oracle_block_manager.py`` to closed forms, library routines,
invariants the pages state, and the pages' own block-table example.
"""
from . import block_manager, cache_ops, fp8, paged_attention, prefill  # noqa: F401
