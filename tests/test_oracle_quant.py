"""Pins for the oracle's quantiser, checked against exact rational arithmetic
and brute force rather than against itself.

The quantiser follows the KV4-RL review (sec. 3, "calibration-free INT4 KV
cache" plus INT8 side cache) with the build's stated readings: symmetric
codes, scale = fp16 rounded toward +inf of max|x|/qmax, codes rounded to
nearest-even.
"""
import bisect
from fractions import Fraction

import numpy as np
import pytest

import oracle as O


def _bf16_value(bits):
    return float(np.array([int(bits) << 16], np.uint32).view(np.float32)[0])


def _to_bf16_bits(x):
    """float -> nearest bf16 bits (only used on values that are exact in bf16)."""
    u = np.array([x], np.float32).view(np.uint32)[0]
    assert u & 0xFFFF == 0, x
    return int(u >> 16)


_FP16 = None


def _fp16_table():
    global _FP16
    if _FP16 is None:
        bits = np.arange(1, 0x7C00, dtype=np.uint16)
        vals = [Fraction(float(v)) for v in bits.view(np.float16)]
        _FP16 = (vals, bits)
    return _FP16


def _exact_ru_fp16(y: Fraction):
    vals, bits = _fp16_table()
    if y == 0:
        return 0
    i = bisect.bisect_left(vals, y)
    return None if i == len(vals) else int(bits[i])


@pytest.mark.parametrize("qmax,quant", [(7, O.quant_int4), (127, O.quant_int8)])
def test_scale_exhaustive_over_bf16(qmax, quant):
    """Every positive finite bf16 group maximum: scale bits == exact RU_fp16(a/qmax)."""
    n = 32 if qmax == 7 else 128
    x = np.zeros(n, np.uint16)
    mismatches = []
    for bits in range(1, 0x7F80):
        x[5] = bits
        sc, codes, ov = quant(x)
        y = Fraction(_bf16_value(bits)) / qmax
        want = _exact_ru_fp16(y)
        if want is None:
            ok = (ov == 1 and sc == 0x7BFF)
        else:
            ok = (ov == 0 and sc == want)
        if not ok:
            mismatches.append((bits, sc, want, ov))
    assert not mismatches, mismatches[:10]


def _brute_code(x: Fraction, s: Fraction, qmax):
    best = None
    for k in range(-qmax, qmax + 1):
        d = abs(x - k * s)
        if best is None or d < best[0] or (d == best[0] and k % 2 == 0):
            best = (d, k)
    return best[1]


@pytest.mark.parametrize("qmax,quant,n", [(7, O.quant_int4, 32), (127, O.quant_int8, 64)])
def test_codes_brute_force(qmax, quant, n):
    """Each code minimises |x - k*s| over the code range, ties to the even k."""
    rng = np.random.default_rng(7)
    for trial in range(300):
        scale = 10.0 ** rng.uniform(-6, 3)
        vals = (rng.standard_normal(n) * scale).astype(np.float32)
        bits = (vals.view(np.uint32) >> 16).astype(np.uint16)   # truncation: some bf16 value
        sc, codes, ov = quant(bits)
        assert ov == 0
        s = Fraction(O.fp16_to_float(sc))
        for i in range(n):
            x = Fraction(_bf16_value(bits[i]))
            assert codes[i] == _brute_code(x, s, qmax), (trial, i)


def test_ties_round_to_even():
    # group max 7 -> s = RU(7/7) = 1 exactly; x = k + 1/2 are bf16-exact ties.
    x = np.zeros(32, np.uint16)
    vals = [7.0, 2.5, 3.5, 0.5, 1.5, -0.5, -1.5, -2.5, 6.5, -6.5, 4.5, -3.5]
    for i, v in enumerate(vals):
        x[i] = _to_bf16_bits(v)
    sc, codes, ov = O.quant_int4(x)
    assert sc == 0x3C00 and ov == 0
    assert list(codes[: len(vals)]) == [7, 2, 4, 0, 2, 0, -2, -2, 6, -6, 4, -4]


def test_invariants_and_requantisation():
    rng = np.random.default_rng(11)
    for _ in range(200):
        vals = (rng.standard_normal(32) * 10.0 ** rng.uniform(-4, 4)).astype(np.float32)
        bits = (vals.view(np.uint32) >> 16).astype(np.uint16)
        sc, codes, _ = O.quant_int4(bits)
        s = O.fp16_to_float(sc)
        assert np.all(np.abs(codes) <= 7)
        xs = np.array([_bf16_value(b) for b in bits])
        assert np.all(np.abs(xs - codes * s) <= s / 2)         # error <= s/2
    # values k * 2^e with max 7 * 2^e: s = 2^e exactly, codes return k
    for e in (-20, -3, 0, 5):
        ks = np.array([7, -7, 0, 3, -2, 5, 1, -6] * 4)
        bits = np.array([_to_bf16_bits(float(k) * 2.0 ** e) for k in ks], np.uint16)
        sc, codes, _ = O.quant_int4(bits)
        assert O.fp16_to_float(sc) == 2.0 ** e
        assert np.array_equal(codes, ks)
    # a group of +-a only: codes are +-7
    a = _to_bf16_bits(3.140625)
    bits = np.array([a if i % 3 else a | 0x8000 for i in range(32)], np.uint16)
    _, codes, _ = O.quant_int4(bits)
    assert set(np.abs(codes).tolist()) == {7}
    # all-zero group: scale 0, codes 0
    sc, codes, _ = O.quant_int4(np.zeros(32, np.uint16))
    assert sc == 0 and not codes.any()


def test_fp16_decoder_against_numpy():
    bits = np.arange(0, 0x7C00, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([O.fp16_to_float(int(b)) for b in bits[::97]])
    assert np.array_equal(got, ref[::97])


def test_overflow_flag():
    # |x| = 2^19 -> a/7 = 74898 > 65504: scale saturates to 0x7BFF and the flag is set
    x = np.zeros(32, np.uint16)
    x[0] = _to_bf16_bits(2.0 ** 19)
    x[1] = _to_bf16_bits(-(2.0 ** 18))
    sc, codes, ov = O.quant_int4(x)
    assert ov == 1 and sc == 0x7BFF and codes[0] == 7 and codes[1] == -4
