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
    vals = (bits << 16).view(np.float32).astype(np.float64)
    return vals[np.isfinite(vals)]


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
