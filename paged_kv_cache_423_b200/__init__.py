"""Python binding of libpkv.so, the B200 paged KV-cache decode library.

A thin ctypes layer with the same names as the C ABI in ``include/pkv.h``: it
checks tensor shapes/dtypes, passes raw pointers, sizes and the current CUDA
stream, and turns return codes into exceptions.  Every step of the decode path
runs in the library's kernels; nothing here computes.  If the library has not
been built, importing the binding's entry points raises -- there is no fallback.

PyTorch provides device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = [
    "PKV_OK", "PKV_ERR_INVALID", "PKV_ERR_OOM", "PKV_ERR_CUDA", "PKV_ERR_UNSUPPORTED",
    "PKV_DEV_BAD_SLOT", "PKV_DEV_BAD_BLOCK", "PKV_DEV_BAD_CONTEXT", "PKV_DEV_BAD_PAIR", "PKV_DEV_TIMEOUT",
    "PATH_AUTO", "PATH_SIMT", "PATH_TENSOR", "PkvError", "library", "library_path",
    "reshape_and_cache", "copy_blocks", "paged_attention_workspace_size", "paged_attention_partition_tokens",
    "paged_attention_decode", "paged_attention_decode_static", "STATIC_SCRATCH_BYTES",
    "paged_attention_prefill_workspace_size", "paged_attention_prefill", "reshape_and_cache_fp8",
    "paged_attention_decode_fp8", "swap_blocks", "BlockManager", "stream_read",
    "SharedPlanInfo", "shared_plan", "paged_attention_decode_shared_workspace_size", "paged_attention_decode_shared",
    "paged_attention_decode_shared_fp8_workspace_size", "paged_attention_decode_shared_fp8",
]

PKV_OK = 0
PKV_ERR_INVALID = -1
PKV_ERR_OOM = -2
PKV_ERR_CUDA = -3
PKV_ERR_UNSUPPORTED = -4
PKV_DEV_BAD_SLOT = 0x1
PKV_DEV_BAD_BLOCK = 0x2
PKV_DEV_BAD_CONTEXT = 0x4
PKV_DEV_BAD_PAIR = 0x8
PKV_DEV_TIMEOUT = 0x10
PATH_AUTO, PATH_SIMT, PATH_TENSOR = 0, 1, 2
DTYPE_BF16, DTYPE_F32 = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    """The in-tree libpkv.so, or the build named by the PKV_LIBRARY environment variable
    (another build of the same sources, e.g. the one-stage-ring variant a test compares)."""
    return os.environ.get("PKV_LIBRARY") or os.path.join(_HERE, "libpkv.so")


class PkvError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


_lib = None

c_int, c_int64, c_size_t, c_float, c_void_p = ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float, ctypes.c_void_p
P_i32 = ctypes.POINTER(ctypes.c_int32)
P_i64 = ctypes.POINTER(ctypes.c_int64)

_SIGNATURES = {
    "pkv_last_error_string": (ctypes.c_char_p, []),
    "pkv_version": (c_int, []),
    "pkv_reshape_and_cache": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
                                      c_int, c_void_p, c_void_p]),
    "pkv_copy_blocks": (c_int, [ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p), c_int, c_void_p, c_int, c_int,
                                c_int64, c_void_p, c_void_p]),
    "pkv_paged_attention_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int, c_int]),
    "pkv_paged_attention_partition_tokens": (c_int, [c_int, c_int, c_int, c_int]),
    "pkv_paged_attention_decode": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p,
                                           c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_float, c_int, c_int,
                                           c_void_p, c_size_t, c_void_p, c_void_p]),
    "pkv_paged_attention_decode_static": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                                  c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_float,
                                                  c_int, c_int, c_void_p, c_void_p]),
    "pkv_paged_attention_prefill_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int]),
    "pkv_paged_attention_prefill": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                            c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                            c_int, c_float, c_void_p, c_size_t, c_void_p, c_void_p]),
    "pkv_reshape_and_cache_fp8": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                          c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p]),
    "pkv_paged_attention_decode_fp8": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                               c_void_p, c_int, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                               c_int, c_float, c_int, c_int, c_void_p, c_size_t, c_void_p,
                                               c_void_p]),
    "pkv_swap_blocks": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int64, c_void_p, c_void_p]),
    "pkv_stream_read": (c_int, [c_void_p, c_size_t, c_void_p, c_void_p]),
    "pkv_bm_create": (c_void_p, [c_int, c_int, c_void_p]),
    "pkv_bm_create_with_swap_space": (c_void_p, [c_int, c_int, c_void_p, c_int]),
    "pkv_bm_num_host_free": (c_int, [c_void_p]),
    "pkv_bm_host_refcount": (c_int, [c_void_p, ctypes.c_int32]),
    "pkv_bm_is_swapped": (c_int, [c_void_p, c_int64]),
    "pkv_bm_swap_out": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_int, ctypes.POINTER(c_int)]),
    "pkv_bm_swap_in": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_int, ctypes.POINTER(c_int)]),
    "pkv_bm_add_seq_tokens": (c_int, [c_void_p, c_int64, c_void_p, c_int, ctypes.POINTER(c_int)]),
    "pkv_bm_num_cached_blocks": (c_int, [c_void_p]),
    "pkv_bm_destroy": (None, [c_void_p]),
    "pkv_bm_num_blocks": (c_int, [c_void_p]),
    "pkv_bm_block_size": (c_int, [c_void_p]),
    "pkv_bm_num_free": (c_int, [c_void_p]),
    "pkv_bm_free_list": (c_int, [c_void_p, c_void_p, c_int]),
    "pkv_bm_alloc": (c_int, [c_void_p, P_i32]),
    "pkv_bm_incref": (c_int, [c_void_p, ctypes.c_int32]),
    "pkv_bm_decref": (c_int, [c_void_p, ctypes.c_int32]),
    "pkv_bm_refcount": (c_int, [c_void_p, ctypes.c_int32]),
    "pkv_bm_add_seq": (c_int, [c_void_p, c_int64, c_int, c_void_p, c_int]),
    "pkv_bm_fork": (c_int, [c_void_p, c_int64, c_int64]),
    "pkv_bm_append_slots": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_void_p, ctypes.POINTER(c_int)]),
    "pkv_bm_append_tokens": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_void_p, ctypes.POINTER(c_int)]),
    "pkv_bm_slots": (c_int, [c_void_p, c_int64, c_int, c_int, c_void_p]),
    "pkv_bm_free_seq": (c_int, [c_void_p, c_int64]),
    "pkv_bm_seq_len": (c_int, [c_void_p, c_int64]),
    "pkv_bm_seq_blocks": (c_int, [c_void_p, c_int64]),
    "pkv_bm_export_tables": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_int, c_void_p]),
}


def _id_array(seq_ids) -> np.ndarray:
    """Sequence ids as a contiguous int64 array (an int64 array is used as it is; any other
    iterable is read once)."""
    if isinstance(seq_ids, np.ndarray) and seq_ids.dtype == np.int64 and seq_ids.flags.c_contiguous:
        return seq_ids
    return np.ascontiguousarray(seq_ids if isinstance(seq_ids, (np.ndarray, list, tuple)) else list(seq_ids),
                                dtype=np.int64)


class SharedPlanInfo(ctypes.Structure):
    """pkv_shared_plan_info: counts and byte offsets of a shared-prefix plan."""
    _fields_ = [(n, ctypes.c_int32) for n in ("num_seqs", "num_segments", "num_parts", "num_entries", "num_partials",
                                               "max_suffix_len", "key_chunk", "group", "block_size",
                                               "max_blocks_per_seq")] + \
               [("shared_row_tokens", ctypes.c_int64), ("shared_tokens", ctypes.c_int64)] + \
               [(n, ctypes.c_uint64) for n in ("off_entries", "off_parts", "off_suffix_lens", "off_block_offset",
                                                "off_row_start", "off_row_ids", "bytes")]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


_SIGNATURES["pkv_shared_plan"] = (c_int, [c_void_p, c_int, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                          c_void_p, c_size_t, ctypes.POINTER(SharedPlanInfo)])
_SIGNATURES["pkv_paged_attention_decode_shared_workspace_size"] = (c_size_t, [ctypes.POINTER(SharedPlanInfo), c_int,
                                                                              c_int, c_int])
_SIGNATURES["pkv_paged_attention_decode_shared"] = (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                                            c_int, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                                            c_float, c_void_p, ctypes.POINTER(SharedPlanInfo),
                                                            c_void_p, c_size_t, c_void_p, c_void_p])
_SIGNATURES["pkv_paged_attention_decode_shared_fp8_workspace_size"] = (c_size_t, [ctypes.POINTER(SharedPlanInfo),
                                                                                  c_int, c_int, c_int])
_SIGNATURES["pkv_paged_attention_decode_shared_fp8"] = (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                                                                c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_int,
                                                                c_int, c_int, c_int, c_int, c_int, c_float, c_void_p,
                                                                ctypes.POINTER(SharedPlanInfo), c_void_p, c_size_t,
                                                                c_void_p, c_void_p])


def library():
    """Load libpkv.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing; build it with `python -m paged_kv_cache_423_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(rc: int, what: str):
    if rc != PKV_OK:
        raise PkvError(rc, f"{what}: {library().pkv_last_error_string().decode()}")
    return rc


# ---------------------------------------------------------------------------
# torch plumbing: pointers and streams only
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _ptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return c_void_p(t.data_ptr())


def _same_device(what, *tensors):
    """The library launches on the current device, so every CUDA tensor of one call must
    live there (pinned host tensors, where a call takes them, are exempt)."""
    cur = None
    for t in tensors:
        if t is None or not getattr(t, "is_cuda", False):
            continue
        if cur is None:
            cur = _torch().cuda.current_device()
        if t.device.index != cur:
            raise ValueError(f"{what}: every CUDA tensor must be on the current device cuda:{cur}, got {t.device}")


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


# ---------------------------------------------------------------------------
# Kernels
# ---------------------------------------------------------------------------

def reshape_and_cache(key, value, key_cache, value_cache, slot_mapping, status=None, stream=None):
    """Write key/value [T, Hkv, D] bf16 into the pools [NB, Hkv, bs, D] at slot_mapping [T] int64."""
    torch = _torch()
    _same_device("reshape_and_cache", key, value, key_cache, value_cache, slot_mapping, status)
    T, Hkv, D = key.shape
    NB, Hkv2, bs, D2 = key_cache.shape
    if value.shape != key.shape or value_cache.shape != key_cache.shape or (Hkv, D) != (Hkv2, D2):
        raise ValueError("reshape_and_cache: shape mismatch")
    if slot_mapping.shape != (T,):
        raise ValueError("reshape_and_cache: slot_mapping must be [T]")
    rc = library().pkv_reshape_and_cache(
        _ptr(key, torch.bfloat16, "key"), _ptr(value, torch.bfloat16, "value"),
        _ptr(key_cache, torch.bfloat16, "key_cache"), _ptr(value_cache, torch.bfloat16, "value_cache"),
        _ptr(slot_mapping, torch.int64, "slot_mapping"), T, NB, Hkv, D, bs,
        _ptr(status, torch.int32, "status"), _stream(stream))
    _check(rc, "reshape_and_cache")


def copy_blocks(key_caches, value_caches, block_mapping, status=None, stream=None):
    """Copy (src, dst) blocks of block_mapping [n, 2] int64 in every layer's K and V pool.

    Pools are bf16 or 8-bit (uint8 e4m3 codes), all of one dtype and shape; the copy is
    bytewise, so an 8-bit pool passes its block bytes as half as many 2-byte elements."""
    torch = _torch()
    if len(key_caches) != len(value_caches):
        raise ValueError("copy_blocks: layer count mismatch")
    n = int(block_mapping.shape[0]) if block_mapping.numel() else 0
    if block_mapping.numel() and tuple(block_mapping.shape) != (n, 2):
        raise ValueError("copy_blocks: block_mapping must be [n, 2]")
    if not key_caches:
        return
    dtype = key_caches[0].dtype
    if dtype not in (torch.bfloat16, torch.uint8):
        raise TypeError(f"copy_blocks: pools must be bf16 or uint8 (e4m3 codes), got {dtype}")
    NB = key_caches[0].shape[0]
    block_bytes = int(np.prod(key_caches[0].shape[1:])) * key_caches[0].element_size()
    if block_bytes % 16:
        raise ValueError("copy_blocks: a block must be a multiple of 16 bytes")
    block_elems = block_bytes // 2
    for kc, vc in zip(key_caches, value_caches):
        if kc.shape != key_caches[0].shape or vc.shape != key_caches[0].shape:
            raise ValueError("copy_blocks: every pool must have the same shape")
    _same_device("copy_blocks", *key_caches, *value_caches, block_mapping, status)
    ks = (c_void_p * len(key_caches))(*[_ptr(k, dtype, "key_cache").value for k in key_caches])
    vs = (c_void_p * len(value_caches))(*[_ptr(v, dtype, "value_cache").value for v in value_caches])
    mapping = _ptr(block_mapping, torch.int64, "block_mapping") if n else c_void_p(0)
    rc = library().pkv_copy_blocks(ks, vs, len(key_caches), mapping, n, NB, block_elems,
                                   _ptr(status, torch.int32, "status"), _stream(stream))
    _check(rc, "copy_blocks")


def paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_context_len,
                                   partition_tokens=0) -> int:
    n = library().pkv_paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                     max_context_len, partition_tokens)
    if n == 0:
        raise PkvError(PKV_ERR_INVALID, "paged_attention_workspace_size: bad arguments")
    return int(n)


def paged_attention_partition_tokens(num_seqs, num_kv_heads, block_size, max_context_len) -> int:
    r = library().pkv_paged_attention_partition_tokens(num_seqs, num_kv_heads, block_size, max_context_len)
    if r < 0:
        _check(r, "paged_attention_partition_tokens")
    return int(r)


def paged_attention_decode(out, query, key_cache, value_cache, block_tables, context_lens, max_context_len, scale,
                           workspace, partition_tokens=0, path=PATH_AUTO, status=None, stream=None):
    """Decode attention: out [B, Hq, D] (bf16 or f32) from query [B, Hq, D] bf16 over the paged pools.

    block_tables [B, max_blocks] int32, context_lens [B] int32 (device), max_context_len
    a host bound, workspace a uint8 device tensor of paged_attention_workspace_size bytes."""
    torch = _torch()
    _same_device("paged_attention_decode", out, query, key_cache, value_cache, block_tables, context_lens, workspace, status)
    B, Hq, D = query.shape
    NB, Hkv, bs, D2 = key_cache.shape
    if out.shape != query.shape or D2 != D or value_cache.shape != key_cache.shape:
        raise ValueError("paged_attention_decode: shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or tuple(context_lens.shape) != (B,):
        raise ValueError("paged_attention_decode: block_tables must be [B, max_blocks], context_lens [B]")
    if out.dtype == torch.bfloat16:
        out_dtype = DTYPE_BF16
    elif out.dtype == torch.float32:
        out_dtype = DTYPE_F32
    else:
        raise TypeError("paged_attention_decode: out must be bf16 or f32")
    rc = library().pkv_paged_attention_decode(
        _ptr(out, None, "out"), out_dtype, _ptr(query, torch.bfloat16, "query"),
        _ptr(key_cache, torch.bfloat16, "key_cache"), _ptr(value_cache, torch.bfloat16, "value_cache"),
        _ptr(block_tables, torch.int32, "block_tables"), int(block_tables.shape[1]),
        _ptr(context_lens, torch.int32, "context_lens"), int(max_context_len), B, Hq, Hkv, D, bs, NB,
        float(scale), int(partition_tokens), int(path), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _ptr(status, torch.int32, "status"), _stream(stream))
    _check(rc, "paged_attention_decode")


STATIC_SCRATCH_BYTES = 64 * 1024 * 1024


def paged_attention_decode_static(out, query, key_cache, value_cache, block_tables, context_lens, max_context_len,
                                  scale, partition_tokens=0, path=PATH_AUTO, status=None, stream=None):
    """paged_attention_decode without a workspace, for callers that cannot allocate
    device memory: the scratch is a fixed array inside the library (STATIC_SCRATCH_BYTES
    per GPU).  Calls on one device must not overlap on the GPU; the first call on a
    device should come before any stream capture."""
    torch = _torch()
    _same_device("paged_attention_decode_static", out, query, key_cache, value_cache, block_tables, context_lens, status)
    B, Hq, D = query.shape
    NB, Hkv, bs, D2 = key_cache.shape
    if out.shape != query.shape or D2 != D or value_cache.shape != key_cache.shape:
        raise ValueError("paged_attention_decode_static: shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or tuple(context_lens.shape) != (B,):
        raise ValueError("paged_attention_decode_static: block_tables must be [B, max_blocks], context_lens [B]")
    out_dtype = {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_F32}.get(out.dtype)
    if out_dtype is None:
        raise TypeError("paged_attention_decode_static: out must be bf16 or f32")
    rc = library().pkv_paged_attention_decode_static(
        _ptr(out, None, "out"), out_dtype, _ptr(query, torch.bfloat16, "query"),
        _ptr(key_cache, torch.bfloat16, "key_cache"), _ptr(value_cache, torch.bfloat16, "value_cache"),
        _ptr(block_tables, torch.int32, "block_tables"), int(block_tables.shape[1]),
        _ptr(context_lens, torch.int32, "context_lens"), int(max_context_len), B, Hq, Hkv, D, bs, NB,
        float(scale), int(partition_tokens), int(path), _ptr(status, torch.int32, "status"), _stream(stream))
    _check(rc, "paged_attention_decode_static")


def reshape_and_cache_fp8(key, value, key_cache, value_cache, slot_mapping, k_scale, v_scale, status=None,
                          stream=None):
    """Quantising write of key/value [T, Hkv, D] bf16 into 8-bit pools [NB, Hkv, bs, D] uint8
    (e4m3 codes) with per-kv-head float32 scales k_scale, v_scale [Hkv]."""
    torch = _torch()
    _same_device("reshape_and_cache_fp8", key, value, key_cache, value_cache, slot_mapping, k_scale, v_scale, status)
    T, Hkv, D = key.shape
    NB, Hkv2, bs, D2 = key_cache.shape
    if value.shape != key.shape or value_cache.shape != key_cache.shape or (Hkv, D) != (Hkv2, D2):
        raise ValueError("reshape_and_cache_fp8: shape mismatch")
    if slot_mapping.shape != (T,) or tuple(k_scale.shape) != (Hkv,) or tuple(v_scale.shape) != (Hkv,):
        raise ValueError("reshape_and_cache_fp8: slot_mapping must be [T], scales [Hkv]")
    rc = library().pkv_reshape_and_cache_fp8(
        _ptr(key, torch.bfloat16, "key"), _ptr(value, torch.bfloat16, "value"),
        _ptr(key_cache, torch.uint8, "key_cache"), _ptr(value_cache, torch.uint8, "value_cache"),
        _ptr(slot_mapping, torch.int64, "slot_mapping"), _ptr(k_scale, torch.float32, "k_scale"),
        _ptr(v_scale, torch.float32, "v_scale"), T, NB, Hkv, D, bs, _ptr(status, torch.int32, "status"),
        _stream(stream))
    _check(rc, "reshape_and_cache_fp8")


def paged_attention_decode_fp8(out, query, key_cache, value_cache, k_scale, v_scale, block_tables, context_lens,
                               max_context_len, scale, workspace, partition_tokens=0, path=PATH_AUTO, status=None,
                               stream=None):
    """Decode attention over 8-bit pools [NB, Hkv, bs, 128] uint8 with per-kv-head scales;
    otherwise as paged_attention_decode (same workspace size).  path: PATH_AUTO (tensor
    cores for 2 <= group <= 16), PATH_SIMT or PATH_TENSOR."""
    torch = _torch()
    _same_device("paged_attention_decode_fp8", out, query, key_cache, value_cache, k_scale, v_scale, block_tables,
                 context_lens, workspace, status)
    B, Hq, D = query.shape
    NB, Hkv, bs, D2 = key_cache.shape
    if out.shape != query.shape or D2 != D or value_cache.shape != key_cache.shape:
        raise ValueError("paged_attention_decode_fp8: shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or tuple(context_lens.shape) != (B,):
        raise ValueError("paged_attention_decode_fp8: block_tables must be [B, max_blocks], context_lens [B]")
    out_dtype = {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_F32}.get(out.dtype)
    if out_dtype is None:
        raise TypeError("paged_attention_decode_fp8: out must be bf16 or f32")
    rc = library().pkv_paged_attention_decode_fp8(
        _ptr(out, None, "out"), out_dtype, _ptr(query, torch.bfloat16, "query"),
        _ptr(key_cache, torch.uint8, "key_cache"), _ptr(value_cache, torch.uint8, "value_cache"),
        _ptr(k_scale, torch.float32, "k_scale"), _ptr(v_scale, torch.float32, "v_scale"),
        _ptr(block_tables, torch.int32, "block_tables"), int(block_tables.shape[1]),
        _ptr(context_lens, torch.int32, "context_lens"), int(max_context_len), B, Hq, Hkv, D, bs, NB,
        float(scale), int(partition_tokens), int(path), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _ptr(status, torch.int32, "status"), _stream(stream))
    _check(rc, "paged_attention_decode_fp8")


def _any_ptr(t, name):
    """Pointer of a contiguous tensor in device memory or pinned host memory."""
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda and not t.is_pinned():
        raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")
    return c_void_p(t.data_ptr())


def swap_blocks(src_pool, dst_pool, block_mapping, status=None, stream=None):
    """Copy blocks between pools [NB, ...] (device and/or pinned host, same block shape and
    dtype): dst_pool[d] = src_pool[s] for every (s, d) of block_mapping [n, 2] int64 (device or
    pinned host).  One kernel launch."""
    torch = _torch()
    _same_device("swap_blocks", src_pool, dst_pool, block_mapping, status)
    if src_pool.dtype != dst_pool.dtype or src_pool.shape[1:] != dst_pool.shape[1:]:
        raise ValueError("swap_blocks: pools must share dtype and block shape")
    n = int(block_mapping.shape[0]) if block_mapping.numel() else 0
    if block_mapping.numel() and (tuple(block_mapping.shape) != (n, 2) or block_mapping.dtype != torch.int64):
        raise ValueError("swap_blocks: block_mapping must be [n, 2] int64")
    if n == 0:
        return
    block_bytes = int(np.prod(src_pool.shape[1:])) * src_pool.element_size()
    rc = library().pkv_swap_blocks(_any_ptr(src_pool, "src_pool"), _any_ptr(dst_pool, "dst_pool"),
                                   _any_ptr(block_mapping, "block_mapping"), n, int(src_pool.shape[0]),
                                   int(dst_pool.shape[0]), block_bytes, _ptr(status, torch.int32, "status"),
                                   _stream(stream))
    _check(rc, "swap_blocks")


def stream_read(buf, sink, stream=None):
    """Read the contiguous device tensor `buf` once, XOR-folding its 32-bit words into
    sink (a 1-element int32 device tensor, set by the caller).  A bandwidth reference."""
    torch = _torch()
    _same_device("stream_read", buf, sink)
    nbytes = buf.numel() * buf.element_size()
    rc = library().pkv_stream_read(_ptr(buf, None, "buf"), nbytes, _ptr(sink, torch.int32, "sink"), _stream(stream))
    _check(rc, "stream_read")


def paged_attention_prefill_workspace_size(num_seqs, total_q, num_heads, num_kv_heads) -> int:
    n = library().pkv_paged_attention_prefill_workspace_size(num_seqs, total_q, num_heads, num_kv_heads)
    if n == 0:
        raise PkvError(PKV_ERR_INVALID, "paged_attention_prefill_workspace_size: bad arguments")
    return int(n)


def paged_attention_prefill(out, query, key_cache, value_cache, block_tables, query_start, context_lens,
                            max_context_len, scale, workspace, status=None, stream=None):
    """Causal prefill / chunked-prefill attention: out [T, Hq, 128] (bf16 or f32) from the
    packed query rows [T, Hq, 128] bf16 of every sequence's new tokens.

    query_start [B+1] int32 and context_lens [B] int32 (device), max_context_len a host
    bound, workspace a uint8 device tensor of paged_attention_prefill_workspace_size bytes."""
    torch = _torch()
    _same_device("paged_attention_prefill", out, query, key_cache, value_cache, block_tables, query_start, context_lens,
                 workspace, status)
    T, Hq, D = query.shape
    NB, Hkv, bs, D2 = key_cache.shape
    B = int(context_lens.shape[0])
    if out.shape != query.shape or D2 != D or value_cache.shape != key_cache.shape:
        raise ValueError("paged_attention_prefill: shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or tuple(query_start.shape) != (B + 1,):
        raise ValueError("paged_attention_prefill: block_tables must be [B, max_blocks], query_start [B+1]")
    out_dtype = {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_F32}.get(out.dtype)
    if out_dtype is None:
        raise TypeError("paged_attention_prefill: out must be bf16 or f32")
    rc = library().pkv_paged_attention_prefill(
        _ptr(out, None, "out"), out_dtype, _ptr(query, torch.bfloat16, "query"),
        _ptr(key_cache, torch.bfloat16, "key_cache"), _ptr(value_cache, torch.bfloat16, "value_cache"),
        _ptr(block_tables, torch.int32, "block_tables"), int(block_tables.shape[1]),
        _ptr(query_start, torch.int32, "query_start"), _ptr(context_lens, torch.int32, "context_lens"), B, T,
        int(max_context_len), Hq, Hkv, D, bs, NB, float(scale), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _ptr(status, torch.int32, "status"), _stream(stream))
    _check(rc, "paged_attention_prefill")


# ---------------------------------------------------------------------------
# Host block manager
# ---------------------------------------------------------------------------

def shared_plan(block_tables, context_lens, num_heads, num_kv_heads, block_size, min_rows=2, key_chunk=0, out=None):
    """Host plan of the shared-prefix decode from host tables [B, max_blocks] int32 and lengths
    [B] int32 (NumPy).  Returns (plan, info): plan a uint8 NumPy array of info.bytes bytes to
    copy to the device, info a SharedPlanInfo.  With `out` (a contiguous uint8 NumPy array, for
    example a view of pinned memory) the plan is written there in one call and a view of its
    first info.bytes bytes is returned; too small a buffer raises."""
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    if tables.ndim != 2 or lens.shape != (tables.shape[0],):
        raise ValueError("shared_plan: block_tables must be [B, max_blocks], context_lens [B]")
    B, mb = tables.shape
    info = SharedPlanInfo()
    lib = library()
    if out is not None:
        if out.dtype != np.uint8 or out.ndim != 1 or not out.flags.c_contiguous:
            raise ValueError("shared_plan: out must be a contiguous 1-D uint8 array")
        _check(lib.pkv_shared_plan(_np_ptr(tables), mb, _np_ptr(lens), B, num_heads, num_kv_heads, block_size,
                                   min_rows, key_chunk, _np_ptr(out), out.nbytes, ctypes.byref(info)), "shared_plan")
        return out[:int(info.bytes)], info
    _check(lib.pkv_shared_plan(_np_ptr(tables), mb, _np_ptr(lens), B, num_heads, num_kv_heads, block_size, min_rows,
                               key_chunk, None, 0, ctypes.byref(info)), "shared_plan")
    plan = np.zeros(int(info.bytes), np.uint8)
    _check(lib.pkv_shared_plan(_np_ptr(tables), mb, _np_ptr(lens), B, num_heads, num_kv_heads, block_size, min_rows,
                               key_chunk, _np_ptr(plan), plan.nbytes, ctypes.byref(info)), "shared_plan")
    return plan, info


def paged_attention_decode_shared_workspace_size(info, num_heads, num_kv_heads, head_dim) -> int:
    return int(library().pkv_paged_attention_decode_shared_workspace_size(ctypes.byref(info), num_heads, num_kv_heads,
                                                                          head_dim))


def paged_attention_decode_shared(out, query, key_cache, value_cache, block_tables, context_lens, scale, plan, info,
                                  workspace, status=None, stream=None):
    """Shared-prefix decode: the result of paged_attention_decode, with blocks that adjacent
    rows share read once per kv head.  plan: the device copy (uint8 tensor) of shared_plan's
    plan for these tables and lengths; info: its SharedPlanInfo."""
    torch = _torch()
    _same_device("paged_attention_decode_shared", out, query, key_cache, value_cache, block_tables, context_lens, plan,
                 workspace, status)
    B, Hq, D = query.shape
    NB, Hkv, bs, D2 = key_cache.shape
    if out.shape != query.shape or D2 != D or value_cache.shape != key_cache.shape:
        raise ValueError("paged_attention_decode_shared: shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or tuple(context_lens.shape) != (B,):
        raise ValueError("paged_attention_decode_shared: block_tables must be [B, max_blocks], context_lens [B]")
    out_dtype = {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_F32}.get(out.dtype)
    if out_dtype is None:
        raise TypeError("paged_attention_decode_shared: out must be bf16 or f32")
    if plan.numel() * plan.element_size() < int(info.bytes):
        raise ValueError("paged_attention_decode_shared: the device plan is smaller than info.bytes")
    rc = library().pkv_paged_attention_decode_shared(
        _ptr(out, None, "out"), out_dtype, _ptr(query, torch.bfloat16, "query"),
        _ptr(key_cache, torch.bfloat16, "key_cache"), _ptr(value_cache, torch.bfloat16, "value_cache"),
        _ptr(block_tables, torch.int32, "block_tables"), int(block_tables.shape[1]),
        _ptr(context_lens, torch.int32, "context_lens"), B, Hq, Hkv, D, bs, NB, float(scale),
        _ptr(plan, torch.uint8, "plan"), ctypes.byref(info), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _ptr(status, torch.int32, "status"), _stream(stream))
    _check(rc, "paged_attention_decode_shared")


def paged_attention_decode_shared_fp8_workspace_size(info, num_heads, num_kv_heads, head_dim) -> int:
    return int(library().pkv_paged_attention_decode_shared_fp8_workspace_size(ctypes.byref(info), num_heads,
                                                                              num_kv_heads, head_dim))


def paged_attention_decode_shared_fp8(out, query, key_cache, value_cache, k_scale, v_scale, block_tables, context_lens,
                                      scale, plan, info, workspace, status=None, stream=None):
    """Shared-prefix decode over 8-bit pools [NB, Hkv, bs, 128] uint8 with per-kv-head scales:
    the result of paged_attention_decode_fp8; otherwise as paged_attention_decode_shared (its
    workspace from paged_attention_decode_shared_fp8_workspace_size)."""
    torch = _torch()
    _same_device("paged_attention_decode_shared_fp8", out, query, key_cache, value_cache, k_scale, v_scale,
                 block_tables, context_lens, plan, workspace, status)
    B, Hq, D = query.shape
    NB, Hkv, bs, D2 = key_cache.shape
    if out.shape != query.shape or D2 != D or value_cache.shape != key_cache.shape:
        raise ValueError("paged_attention_decode_shared_fp8: shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or tuple(context_lens.shape) != (B,):
        raise ValueError("paged_attention_decode_shared_fp8: block_tables must be [B, max_blocks], context_lens [B]")
    out_dtype = {torch.bfloat16: DTYPE_BF16, torch.float32: DTYPE_F32}.get(out.dtype)
    if out_dtype is None:
        raise TypeError("paged_attention_decode_shared_fp8: out must be bf16 or f32")
    if plan.numel() * plan.element_size() < int(info.bytes):
        raise ValueError("paged_attention_decode_shared_fp8: the device plan is smaller than info.bytes")
    rc = library().pkv_paged_attention_decode_shared_fp8(
        _ptr(out, None, "out"), out_dtype, _ptr(query, torch.bfloat16, "query"),
        _ptr(key_cache, torch.uint8, "key_cache"), _ptr(value_cache, torch.uint8, "value_cache"),
        _ptr(k_scale, torch.float32, "k_scale"), _ptr(v_scale, torch.float32, "v_scale"),
        _ptr(block_tables, torch.int32, "block_tables"), int(block_tables.shape[1]),
        _ptr(context_lens, torch.int32, "context_lens"), B, Hq, Hkv, D, bs, NB, float(scale),
        _ptr(plan, torch.uint8, "plan"), ctypes.byref(info), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _ptr(status, torch.int32, "status"), _stream(stream))
    _check(rc, "paged_attention_decode_shared_fp8")


def _np_ptr(a):
    return c_void_p(a.ctypes.data) if a is not None and a.size else c_void_p(0)


class BlockManager:
    """Free list + reference counts + per-sequence block tables (host, C++)."""

    def __init__(self, num_blocks: int, block_size: int, initial_order=None, num_host_blocks: int = 0):
        lib = library()
        order = None if initial_order is None else np.ascontiguousarray(initial_order, dtype=np.int32)
        if order is not None and order.shape != (num_blocks,):
            raise ValueError("initial_order must have num_blocks entries")
        h = lib.pkv_bm_create_with_swap_space(num_blocks, block_size,
                                              _np_ptr(order) if order is not None else None, num_host_blocks)
        if not h:
            raise PkvError(PKV_ERR_INVALID, lib.pkv_last_error_string().decode())
        self._h = c_void_p(h)
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.num_host_blocks = num_host_blocks

    def close(self):
        if getattr(self, "_h", None):
            library().pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def num_free(self) -> int:
        return library().pkv_bm_num_free(self._h)

    def free_list(self) -> list[int]:
        buf = np.zeros(self.num_blocks, np.int32)
        n = library().pkv_bm_free_list(self._h, _np_ptr(buf), self.num_blocks)
        return buf[:n].tolist()

    def alloc(self) -> int:
        b = ctypes.c_int32()
        _check(library().pkv_bm_alloc(self._h, ctypes.byref(b)), "bm_alloc")
        return b.value

    def incref(self, block: int):
        _check(library().pkv_bm_incref(self._h, block), "bm_incref")

    def decref(self, block: int):
        _check(library().pkv_bm_decref(self._h, block), "bm_decref")

    def refcount(self, block: int) -> int:
        r = library().pkv_bm_refcount(self._h, block)
        if r < 0:
            _check(r, "bm_refcount")
        return r

    def add_seq(self, seq_id: int, num_tokens: int, shared_prefix_blocks=()):
        shared = np.ascontiguousarray(list(shared_prefix_blocks), dtype=np.int32)
        _check(library().pkv_bm_add_seq(self._h, seq_id, num_tokens, _np_ptr(shared), len(shared)), "bm_add_seq")

    def fork(self, parent: int, child: int):
        _check(library().pkv_bm_fork(self._h, parent, child), "bm_fork")

    def append_slots(self, seq_ids):
        ids = _id_array(seq_ids)
        slots = np.zeros(len(ids), np.int64)
        pairs = np.zeros((max(len(ids), 1), 2), np.int64)
        n_cow = c_int(0)
        _check(library().pkv_bm_append_slots(self._h, _np_ptr(ids), len(ids), _np_ptr(slots), _np_ptr(pairs),
                                             ctypes.byref(n_cow)), "bm_append_slots")
        return slots, pairs[:n_cow.value].copy()

    def append_tokens(self, seq_ids, tokens):
        """append_slots with the token id of each new position; a sequence created from
        token ids registers every block these tokens complete in the prefix cache."""
        ids = _id_array(seq_ids)
        toks = np.ascontiguousarray(list(tokens), dtype=np.int32)
        if len(toks) != len(ids):
            raise ValueError("append_tokens: one token per sequence")
        slots = np.zeros(len(ids), np.int64)
        pairs = np.zeros((max(len(ids), 1), 2), np.int64)
        n_cow = c_int(0)
        _check(library().pkv_bm_append_tokens(self._h, _np_ptr(ids), _np_ptr(toks), len(ids), _np_ptr(slots),
                                              _np_ptr(pairs), ctypes.byref(n_cow)), "bm_append_tokens")
        return slots, pairs[:n_cow.value].copy()

    def slots(self, seq_id: int, start: int, count: int) -> np.ndarray:
        out = np.zeros(count, np.int64)
        _check(library().pkv_bm_slots(self._h, seq_id, start, count, _np_ptr(out)), "bm_slots")
        return out

    def free_seq(self, seq_id: int):
        _check(library().pkv_bm_free_seq(self._h, seq_id), "bm_free_seq")

    def seq_len(self, seq_id: int) -> int:
        r = library().pkv_bm_seq_len(self._h, seq_id)
        if r < 0:
            _check(r, "bm_seq_len")
        return r

    def seq_blocks(self, seq_id: int) -> int:
        r = library().pkv_bm_seq_blocks(self._h, seq_id)
        if r < 0:
            _check(r, "bm_seq_blocks")
        return r

    def export_tables(self, seq_ids, max_blocks: int):
        ids = _id_array(seq_ids)
        tables = np.zeros((len(ids), max_blocks), np.int32)
        lens = np.zeros(len(ids), np.int32)
        _check(library().pkv_bm_export_tables(self._h, _np_ptr(ids), len(ids), _np_ptr(tables), max_blocks,
                                              _np_ptr(lens)), "bm_export_tables")
        return tables, lens

    # -- swap space ---------------------------------------------------------------
    def num_host_free(self) -> int:
        return library().pkv_bm_num_host_free(self._h)

    def host_refcount(self, block: int) -> int:
        r = library().pkv_bm_host_refcount(self._h, block)
        if r < 0:
            _check(r, "bm_host_refcount")
        return r

    def is_swapped(self, seq_id: int) -> bool:
        r = library().pkv_bm_is_swapped(self._h, seq_id)
        if r < 0:
            _check(r, "bm_is_swapped")
        return bool(r)

    def _swap(self, fn, seq_ids, what):
        ids = _id_array(seq_ids)
        cap = max(self.num_blocks, self.num_host_blocks, 1)
        pairs = np.zeros((cap, 2), np.int64)
        n = c_int(0)
        _check(fn(self._h, _np_ptr(ids), len(ids), _np_ptr(pairs), cap, ctypes.byref(n)), what)
        return pairs[:n.value].copy()

    def swap_out(self, seq_ids) -> np.ndarray:
        """(device, host) block pairs to copy, [n, 2] int64."""
        return self._swap(library().pkv_bm_swap_out, seq_ids, "bm_swap_out")

    def swap_in(self, seq_ids) -> np.ndarray:
        """(host, device) block pairs to copy, [n, 2] int64."""
        return self._swap(library().pkv_bm_swap_in, seq_ids, "bm_swap_in")

    # -- automatic prefix caching ---------------------------------------------------
    def add_seq_tokens(self, seq_id: int, tokens) -> int:
        """New sequence from its prompt token ids; returns the number of leading tokens
        whose K/V are already in the pool (taken from cached blocks)."""
        toks = np.ascontiguousarray(list(tokens), dtype=np.int32)
        cached = c_int(0)
        _check(library().pkv_bm_add_seq_tokens(self._h, seq_id, _np_ptr(toks), len(toks), ctypes.byref(cached)),
               "bm_add_seq_tokens")
        return cached.value

    def num_cached_blocks(self) -> int:
        return library().pkv_bm_num_cached_blocks(self._h)
