"""Number-format facts the 8-bit tensor-core decode relies on, checked exhaustively
with the oracle's e4m3 codec and numpy's IEEE half (no GPU).

* Every bf16 value x with 2^-2 <= |x| < 256 is exactly hi + lo, hi = e4m3(x) and
  lo = e4m3(x - hi) (round to nearest even): the query split loses nothing there.
* Below 2^-2 the split's error is at most half the smallest e4m3 subnormal, 2^-10.
* Every non-negative finite f16 value p <= 2^15 is, within 2^-9 relative (or an
  absolute 2^-17 near zero), the sum of three e5m2 values: hi and mid cut to the top
  byte, lo rounded at its third significant bit; that sum is itself an f16 value.
  e5m2 is the top byte of an f16, so the terms are read off the f16 bit pattern."""
import numpy as np

from oracle.fp8 import E4M3_TABLE, encode_e4m3


def e4m3(x):
    return float(E4M3_TABLE[encode_e4m3(float(x))])


def bf16_values():
    bits = np.arange(1 << 16, dtype=np.uint32)
    finite = (bits & 0x7F80) != 0x7F80           # exponent field not all ones
    return (bits[finite] << 16).view(np.float32).astype(np.float64)


def test_query_split_is_exact_from_a_quarter_up():
    vals = bf16_values()
    sel = vals[(np.abs(vals) >= 0.25) & (np.abs(vals) < 256.0)]
    assert sel.size == 10 * 128 * 2  # 10 binades of 128 mantissas, both signs
    for x in sel:
        hi = e4m3(x)
        assert hi + e4m3(x - hi) == x


def test_query_split_error_below_a_quarter():
    vals = bf16_values()
    sel = vals[np.abs(vals) < 0.25]
    worst = max(abs(x - (e4m3(x) + e4m3(x - e4m3(x)))) for x in sel)
    assert worst <= 2.0 ** -10


def split_p(p16):
    """The three e5m2 terms of a non-negative f16 value, as f16 values, and their sum."""
    def top(v):
        return (np.array(v, np.float16).view(np.uint16) & np.uint16(0xFF00)).view(np.float16)
    hi = top(p16)
    r1 = np.float16(p16 - hi)
    mid = top(r1)
    r2 = np.float16(r1 - mid)
    lo = (np.array(r2, np.float16).view(np.uint16) + np.uint16(0x80) & np.uint16(0xFF00)).view(np.float16)
    total = np.float16(np.float16(hi + mid) + lo)
    return hi, mid, lo, total


def test_softmax_weight_split():
    bits = np.arange(0, 0x7800 + 1, dtype=np.uint16)  # 0 .. 2^15 (all non-negative finite halves up to it)
    p = bits.view(np.float16)
    hi, mid, lo, total = split_p(p)
    exact = hi.astype(np.float64) + mid.astype(np.float64) + lo.astype(np.float64)
    assert np.array_equal(exact, total.astype(np.float64))  # the f16 sum is exact
    err = np.abs(exact - p.astype(np.float64))
    assert np.all(err <= np.maximum(2.0 ** -9 * p.astype(np.float64), 2.0 ** -17))
    for t in (hi, mid, lo):  # each term is an e5m2 value: the low byte of its f16 pattern is zero
        assert np.all((t.view(np.uint16) & 0xFF) == 0)


def emulate_tensor_path(q, keys, values, scale, p_format="e5m2x3"):
    """The 8-bit tensor-core decode's number formats for one head and one item, in NumPy:
    q as e4m3 hi + lo after a power of two that puts max|q| in [128, 256); scores in
    float64 (the MMA accumulates exact e4m3 products in fp32); the held maximum = the
    true maximum; P = 2^(x - m + 7) rounded to f16 and split into the three e5m2 terms
    (or, as a control, P = 2^(x - m) rounded to one e4m3 code); denominators over the
    same represented weights."""
    m = np.abs(q).max()
    e = 0 if m == 0 else 7 - int(np.floor(np.log2(m)))
    x = q * 2.0 ** e
    hi = np.array([e4m3(v) for v in x])
    lo = np.array([e4m3(v - h) for v, h in zip(x, hi)])
    s = keys @ (hi + lo) * 2.0 ** -e
    z = s * scale * np.log2(np.e)
    if p_format == "e5m2x3":
        p = np.exp2(z - z.max() + 7.0).astype(np.float16)
        _, _, _, total = split_p(p)
        w = total.astype(np.float64)
    else:
        w = np.array([e4m3(v) for v in np.exp2(z - z.max())])
    return (w @ values) / w.sum()


def reference(q, keys, values, scale):
    z = keys @ q * scale
    w = np.exp(z - z.max())
    return (w / w.sum()) @ values


def score_cases(rng, q, n, scale):
    """Keys along q with chosen scores (k = a q / |q|^2 gives q.k = a) plus small noise."""
    unit = q / (q @ q)
    noise = lambda: rng.standard_normal((n, q.size)) * 1e-4
    ln2 = np.log(2.0)
    cases = {}
    a = (-12 * ln2 + rng.normal(0, 0.2, n)) / scale             # 2047 weights near 2^-12 of the top:
    a[7] = 0.0                                                    # about a third of the total mass
    cases["dominant_plus_tail"] = a[:, None] * unit + noise()
    a = -rng.uniform(0, 20, n) * ln2 / scale                      # weights spread over 2^-20 .. 1
    cases["deep_tail"] = a[:, None] * unit + noise()
    a = (-14 * ln2 + rng.normal(0, 0.3, n)) / scale
    a[:2] = 0.0, -0.02 / scale                                    # two close modes over a deep tail
    cases["two_modes"] = a[:, None] * unit + noise()
    return cases


def test_split_formats_keep_peaked_attention_in_tolerance():
    """Adversarial score patterns for the weight split: the emulated formats stay within
    the parity tolerance (max-abs 1e-2, relative-L2 5e-3), while P held in one e4m3
    code (weights below 2^-9 of the top lost) misses it on the heavy-tail case."""
    rng = np.random.default_rng(5)
    D, n = 128, 2048
    scale = 1.0 / np.sqrt(D)
    values = rng.standard_normal((n, D))
    q = np.round(rng.standard_normal(D) * 64) / 64
    for name, keys in score_cases(rng, q, n, scale).items():
        ref = reference(q, keys, values, scale)
        got = emulate_tensor_path(q, keys, values, scale)
        assert np.abs(got - ref).max() <= 1e-2, name
        assert np.linalg.norm(got - ref) <= 5e-3 * np.linalg.norm(ref), name
        if name == "dominant_plus_tail":
            bad = emulate_tensor_path(q, keys, values, scale, p_format="e4m3")
            assert np.linalg.norm(bad - ref) > 5e-3 * np.linalg.norm(ref)
