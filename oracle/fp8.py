"""Oracle: an 8-bit (e4m3) KV cache -- the codec, the quantising cache write and
decode attention over the quantised pool.

TEST INFRASTRUCTURE ONLY -- see the package docstring.

What it follows
  * intelliparadigm article, §4.2 (初始化速度慢: loading in low-bit fp8) and §5 (与量化技术
    深度结合; the int4 + vLLM LLaMA-13B example): quantised storage shrinks memory and
    raises throughput.  The pages name fp8 and give no format; the plain reading for a
    KV cache is the e4m3 format defined below, with a float32 scale per kv head.

The e4m3 format (as defined by the OCP 8-bit floating point specification, the
variant without infinities): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
bits.  Exponent field 0 holds the subnormals m/8 * 2^-6; exponent field 1..15
holds (1 + m/8) * 2^(e-7); the pattern S.1111.111 is NaN; the largest finite
magnitude is 448 (S.1111.110).

Readings where the pages are silent (each listed in the design notes):
  * code = e4m3(float32(x) / float32(scale[h])): the division is one correctly rounded
    float32 operation, then round to nearest (ties to even) into e4m3, saturating
    every finite magnitude above 448 to 448; NaN stays NaN.
  * the dequantised value is e4m3_value(code) * scale[h]; attention over the pool is
    the decode attention of the bf16 path applied to those values.

Parity status: pinned (the 256 code values and the rounding of every bf16 value
against torch's float8_e4m3fn conversion; saturation and tie cases worked by hand).
"""
from __future__ import annotations

import math

import numpy as np

from .paged_attention import attend, bf16_bits_to_f64

E4M3_MAX = 448.0
E4M3_NAN = 0x7F


def e4m3_value(code: int) -> float:
    """The real number an e4m3 code stands for (NaN for S.1111.111)."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def encode_e4m3(x: float) -> int:
    """Round one real value to the nearest e4m3 code (ties to even), saturating."""
    if math.isnan(x):
        return E4M3_NAN
    sign = 0x80 if math.copysign(1.0, x) < 0 else 0
    a = abs(x)
    if a == 0.0:
        return sign
    if math.isinf(a):
        return sign | 0x7E                # saturates like every finite overflow
    # spacing of the e4m3 grid around a: 2^(E-3) in binade [2^E, 2^(E+1)), E >= -6;
    # below 2^-6 the subnormal spacing 2^-9
    exp = max(math.frexp(a)[1] - 1, -6)
    quantum = 2.0 ** (exp - 3)
    steps = round(a / quantum)          # exact quotient; Python rounds half to even
    value = steps * quantum
    if value > E4M3_MAX:
        value = E4M3_MAX
    if value == 0.0:
        return sign
    if value < 2.0 ** -6:
        return sign | int(value / 2.0 ** -9)
    mant, e2 = math.frexp(value)        # value = mant * 2^e2, mant in [0.5, 1)
    e = e2 - 1 + 7
    m = int(round((mant * 2.0 - 1.0) * 8))
    return sign | (e << 3) | m


def quantize(x_f32: np.ndarray, scale_f32: float) -> np.ndarray:
    """Codes of float32 values divided (in float32) by a float32 scale."""
    q = (np.asarray(x_f32, np.float32) / np.float32(scale_f32)).astype(np.float32)
    flat = [encode_e4m3(float(v)) for v in q.ravel()]
    return np.array(flat, dtype=np.uint8).reshape(q.shape)


def reshape_and_cache_fp8(key_bits, value_bits, key_cache_codes, value_cache_codes, slot_mapping, k_scale, v_scale):
    """Quantising cache write: token t's K and V (bf16, [T, Hkv, D]) become e4m3 codes
    with the per-kv-head scales and land at slot_mapping[t] (negative = skip).
    Caches [NB, Hkv, bs, D] uint8.  Returns new (key_cache, value_cache)."""
    block_size = key_cache_codes.shape[2]
    num_kv_heads = key_bits.shape[1]
    kc = key_cache_codes.copy()
    vc = value_cache_codes.copy()
    k32 = bf16_bits_to_f64(key_bits).astype(np.float32)
    v32 = bf16_bits_to_f64(value_bits).astype(np.float32)
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64)):
        if slot < 0:
            continue
        block, row = divmod(int(slot), block_size)
        for h in range(num_kv_heads):
            kc[block, h, row, :] = quantize(k32[t, h], k_scale[h])
            vc[block, h, row, :] = quantize(v32[t, h], v_scale[h])
    return kc, vc


def paged_decode_fp8(query_bits, key_cache_codes, value_cache_codes, k_scale, v_scale, block_tables, context_lens,
                     scale):
    """Decode attention over the dequantised pool: float64 [B, Hq, D]."""
    num_seqs, num_heads, head_dim = query_bits.shape
    num_kv_heads = key_cache_codes.shape[1]
    block_size = key_cache_codes.shape[2]
    group = num_heads // num_kv_heads
    scale64 = float(np.float32(scale))
    q_all = bf16_bits_to_f64(query_bits)
    out = np.zeros((num_seqs, num_heads, head_dim), dtype=np.float64)
    for s in range(num_seqs):
        length = int(context_lens[s])
        if length == 0:
            continue
        pos = np.arange(length)
        phys = np.asarray(block_tables[s])[pos // block_size]
        rows = pos % block_size
        for h in range(num_heads):
            kvh = h // group
            keys = e4m3_to_f64(key_cache_codes[phys, kvh, rows, :]) * float(np.float32(k_scale[kvh]))
            values = e4m3_to_f64(value_cache_codes[phys, kvh, rows, :]) * float(np.float32(v_scale[kvh]))
            out[s, h] = attend(q_all[s, h], keys, values, scale64)
    return out
