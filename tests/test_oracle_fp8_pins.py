"""Pins for the 8-bit (e4m3) KV-cache oracle (CPU only).

The codec is tied to torch's float8_e4m3fn type (every one of the 256 code
values; the rounding of every finite bf16 value below the saturation boundary;
float32 division then rounding for non-power-of-two scales), to hand-worked
ties and saturation cases, and the quantised-pool attention to the pinned bf16
decode oracle on pools whose dequantised values are exactly bf16.
"""
import inspect
import math

import numpy as np
import pytest
import torch

import workloads as wl
from oracle import fp8, paged_attention

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


def torch_codes(x_f32):
    return torch.from_numpy(np.ascontiguousarray(x_f32, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def all_bf16_as_f32():
    bits = np.arange(65536, dtype=np.uint32)
    return (bits << 16).view(np.float32)


# ---- codec ------------------------------------------------------------------

def pin_code_values(mod):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([mod.e4m3_value(c) for c in range(256)])
    return np.array_equal(np.isnan(ref), np.isnan(got)) and np.array_equal(ref[~np.isnan(ref)], got[~np.isnan(got)])


def pin_rounding_every_bf16(mod):
    f = all_bf16_as_f32()
    f = f[np.isfinite(f) & (np.abs(f) < 464)]
    got = np.array([mod.encode_e4m3(float(x)) for x in f], np.uint8)
    return np.array_equal(got, torch_codes(f))


def pin_hand_cases(mod):
    cases = {
        1.0: 0x38, 1.0625: 0x38,          # tie between 1.0 (m=0) and 1.125 (m=1): even
        1.1875: 0x3A,                     # tie between 1.125 (m=1) and 1.25 (m=2): even
        2.0 ** -10: 0x00,                 # half the smallest subnormal: tie to even zero
        3 * 2.0 ** -10: 0x02,             # tie between 2^-9 (m=1) and 2^-8 (m=2)
        2.0 ** -6: 0x08,                  # smallest normal
        448.0: 0x7E, 464.0: 0x7E,         # tie between 448 and (unrepresentable) 480: 448
        470.0: 0x7E, 1e30: 0x7E, math.inf: 0x7E,   # saturation
        -448.0: 0xFE, -math.inf: 0xFE, -1.0: 0xB8, -0.0: 0x80,
    }
    return all(mod.encode_e4m3(x) == code for x, code in cases.items()) and mod.encode_e4m3(math.nan) & 0x7F == 0x7F


def pin_quantize_division(mod):
    rng = wl.rng_for(50)
    x = rng.standard_normal(4000).astype(np.float32) * 3
    for scale in (np.float32(1 / 48), np.float32(0.0173), np.float32(3.3)):
        q = (torch.from_numpy(x) / torch.tensor(scale, dtype=torch.float32)).numpy()
        keep = np.abs(q) < 464
        if not np.array_equal(mod.quantize(x, scale)[keep], torch_codes(q[keep])):
            return False
        if not np.all(mod.quantize(x, scale)[~keep] & 0x7F == 0x7E):
            return False
    return True


def pin_table_lookup_every_code(mod):
    """The vectorised lookup e4m3_to_f64 over all 256 codes, laid out as a [2, 8, 16] block, against
    torch's float8_e4m3fn -> float64 conversion (NaN codes stay NaN, the shape is kept)."""
    codes = np.arange(256, dtype=np.uint8).reshape(2, 8, 16)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = mod.e4m3_to_f64(codes)
    nan = np.isnan(ref)
    return got.shape == ref.shape and np.array_equal(nan, np.isnan(got)) and np.array_equal(ref[~nan], got[~nan])


CODEC_PINS = [pin_code_values, pin_rounding_every_bf16, pin_hand_cases, pin_quantize_division, pin_table_lookup_every_code]


@pytest.mark.parametrize("pin", CODEC_PINS, ids=lambda p: p.__name__)
def test_codec_pin(pin):
    assert pin(fp8)


def test_cache_write_matches_element_loop():
    rng = wl.rng_for(51)
    NB, Hkv, bs, D, T = 5, 2, 4, 6, 6
    kc = rng.integers(0, 256, size=(NB, Hkv, bs, D)).astype(np.uint8)
    vc = rng.integers(0, 256, size=(NB, Hkv, bs, D)).astype(np.uint8)
    k = wl.bf16_normal(rng, (T, Hkv, D))
    v = wl.bf16_normal(rng, (T, Hkv, D))
    ks = np.array([0.02, 0.03], np.float32)
    vs = np.array([0.025, 0.015], np.float32)
    slots = np.array([3, -1, 17, 0, 9, 19], np.int64)
    got_k, got_v = fp8.reshape_and_cache_fp8(k, v, kc, vc, slots, ks, vs)
    exp_k, exp_v = kc.copy(), vc.copy()
    kf = (k.astype(np.uint32) << 16).view(np.float32)
    vf = (v.astype(np.uint32) << 16).view(np.float32)
    for t in range(T):
        if slots[t] < 0:
            continue
        for h in range(Hkv):
            for d in range(D):
                exp_k[slots[t] // bs, h, slots[t] % bs, d] = torch_codes(
                    np.array([np.float32(kf[t, h, d]) / ks[h]], np.float32))[0]
                exp_v[slots[t] // bs, h, slots[t] % bs, d] = torch_codes(
                    np.array([np.float32(vf[t, h, d]) / vs[h]], np.float32))[0]
    assert np.array_equal(got_k, exp_k) and np.array_equal(got_v, exp_v)


# ---- attention over the quantised pool ---------------------------------------

def pin_fp8_decode_equals_bf16_decode(impl):
    """Power-of-two scales make every dequantised value an exact bf16 number: the
    8-bit decode must then equal the (pinned) bf16 decode on those values."""
    rng = wl.rng_for(52)
    B, Hq, Hkv, D, bs = 3, 6, 2, 8, 4
    lens = np.array([5, 12, 1], np.int32)
    nb = 12
    tables = wl.place_blocks(lens, bs, rng.permutation(nb).astype(np.int32))
    kc = rng.integers(0, 256, size=(nb, Hkv, bs, D)).astype(np.uint8)
    vc = rng.integers(0, 256, size=(nb, Hkv, bs, D)).astype(np.uint8)
    kc[(kc & 0x7F) == 0x7F] = 0x10      # no NaN codes
    vc[(vc & 0x7F) == 0x7F] = 0x21
    ks = np.array([2.0 ** -5, 2.0 ** -3], np.float32)
    vs = np.array([2.0 ** -4, 2.0 ** -6], np.float32)
    q = wl.bf16_normal(rng, (B, Hq, D))
    kb = wl.f32_to_bf16_bits((fp8.E4M3_TABLE[kc] * ks[None, :, None, None]).astype(np.float32))
    vb = wl.f32_to_bf16_bits((fp8.E4M3_TABLE[vc] * vs[None, :, None, None]).astype(np.float32))
    got = impl(q, kc, vc, ks, vs, tables, lens, 0.3)
    ref = paged_attention.paged_decode(q, kb, vb, tables, lens, 0.3)
    return np.allclose(got, ref, rtol=0, atol=1e-12)


def pin_fp8_decode_single_token(impl):
    rng = wl.rng_for(53)
    lens = np.array([1, 1], np.int32)
    kc = rng.integers(0, 0x70, size=(4, 2, 4, 8)).astype(np.uint8)
    vc = rng.integers(0, 0x70, size=(4, 2, 4, 8)).astype(np.uint8)
    tables = np.array([[2], [0]], np.int32)
    vs = np.array([0.5, 0.25], np.float32)
    got = impl(wl.bf16_normal(rng, (2, 4, 8)), kc, vc, np.array([1.0, 1.0], np.float32), vs, tables, lens, 0.3)
    for s in range(2):
        for h in range(4):
            if not np.array_equal(got[s, h], fp8.E4M3_TABLE[vc[tables[s][0], h // 2, 0]] * vs[h // 2]):
                return False
    return True


DECODE_PINS = [pin_fp8_decode_equals_bf16_decode, pin_fp8_decode_single_token]


@pytest.mark.parametrize("pin", DECODE_PINS, ids=lambda p: p.__name__)
def test_fp8_decode_pin(pin):
    assert pin(fp8.paged_decode_fp8)


def test_quantisation_error_bound():
    """Attention over the 8-bit pool stays close to attention over the bf16 source:
    e4m3 keeps 3 mantissa bits (relative step 2^-3 at most), so with unit-variance
    data the outputs differ by a few percent of their scale, not more."""
    b = wl.make_decode_batch("llama7b", num_seqs=4, length_scale=0.05, num_heads=4, num_kv_heads=2, head_dim=32,
                             block_size=16)
    ks = wl.kv_scales(wl.rng_for(54), 2)
    vs = wl.kv_scales(wl.rng_for(55), 2)
    kf = (b.key_cache.astype(np.uint32) << 16).view(np.float32)
    vf = (b.value_cache.astype(np.uint32) << 16).view(np.float32)
    kc8 = np.stack([fp8.quantize(kf[:, h], ks[h]) for h in range(2)], axis=1)
    vc8 = np.stack([fp8.quantize(vf[:, h], vs[h]) for h in range(2)], axis=1)
    a8 = fp8.paged_decode_fp8(b.query, kc8, vc8, ks, vs, b.block_tables, b.context_lens, b.scale)
    a16 = paged_attention.paged_decode(b.query, b.key_cache, b.value_cache, b.block_tables, b.context_lens, b.scale)
    assert np.max(np.abs(a8 - a16)) < 0.1
    assert np.linalg.norm(a8 - a16) / np.linalg.norm(a16) < 0.06


# ---- mutation tests ------------------------------------------------------------

MUTATIONS = {
    "ties_away_from_zero": ("steps = round(a / quantum)", "steps = math.floor(a / quantum + 0.5)"),
    "no_saturation": ("    if value > E4M3_MAX:\n        value = E4M3_MAX\n", ""),
    "subnormal_floor": ("exp = max(math.frexp(a)[1] - 1, -6)", "exp = max(math.frexp(a)[1] - 1, -7)"),
    "bias_8": ("return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)", "return sign * (1.0 + m / 8.0) * 2.0 ** (e - 8)"),
    "k_scale_for_values": ("* float(np.float32(v_scale[kvh]))", "* float(np.float32(k_scale[kvh]))"),
    "scale_by_query_head": ("* float(np.float32(k_scale[kvh]))", "* float(np.float32(k_scale[h % len(k_scale)]))"),
    "lookup_drops_sign": ("return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]",
                          "return E4M3_TABLE[np.asarray(codes, dtype=np.uint8) & 0x7F]"),
    "multiply_not_divide": ("(np.asarray(x_f32, np.float32) / np.float32(scale_f32))",
                            "(np.asarray(x_f32, np.float32) * np.float32(scale_f32))"),
}


def mutant_module(name):
    old, new = MUTATIONS[name]
    src = inspect.getsource(fp8)
    assert old in src, name
    src = src.replace("from .paged_attention import", "from oracle.paged_attention import")
    ns = {}
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)

    class M:
        pass

    m = M()
    for k, v in ns.items():
        setattr(m, k, v)
    return m


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_fp8_pins_catch_planted_mistake(name):
    m = mutant_module(name)
    caught = []
    for pin in CODEC_PINS:
        try:
            ok = pin(m)
        except Exception:
            ok = False
        if not ok:
            caught.append(pin.__name__)
    for pin in DECODE_PINS:
        try:
            ok = pin(m.paged_decode_fp8)
        except Exception:
            ok = False
        if not ok:
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutation {name}"
