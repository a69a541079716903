"""The checker's own rounding helpers, pinned against exact rational rounding.

``criteria.f64_to_bf16_bits`` and ``criteria.f64_to_f16_bits`` define "round_to_nearest_even(Y)"
for every bf16 / fp16 parity check, and the oracle's ``f32_to_f16_rne`` rounds fp16 results.  A
one-ulp slip in any of them would let a two-ulp GPU error pass, so each is compared here with the
nearest-even rounding computed in exact fractions (``Fraction``), on constructed halfway cases
(exact ties of both parities, one fp64 ulp either side of a tie, the double-rounding trap where
fp32 would round onto a tie first), binade edges, subnormals and random values.
"""
import math
from fractions import Fraction

import numpy as np

import criteria as C
import oracle as O


def _rne_fraction(y: float, mant_bits: int, emin: int) -> Fraction:
    """Nearest value with `mant_bits` significand bits (incl. the implicit one), ties to even, in
    exact rationals; exponents below emin are subnormal (fixed spacing 2^(emin - mant_bits + 1))."""
    if y == 0.0:
        return Fraction(0)
    fy = Fraction(y)
    m, e = math.frexp(abs(y))            # |y| = m * 2^e, 0.5 <= m < 1
    e = max(e - 1, emin)                 # |y| in [2^e, 2^(e+1)) for normals
    ulp = Fraction(2) ** (e - mant_bits + 1)
    q = fy / ulp
    lo = math.floor(q)
    rem = q - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return lo * ulp


def _bf16_bits_of(v: Fraction, y: float) -> int:
    f = np.array([math.copysign(float(v), y)], np.float32)       # a result of 0 keeps y's sign
    assert Fraction(float(f[0])) == v          # exactly representable
    return int(f.view(np.uint32)[0] >> 16)


def _f16_bits_of(v: Fraction, y: float) -> int:
    h = np.array([math.copysign(float(v), y)], np.float16)
    assert Fraction(float(h[0])) == v
    return int(h.view(np.uint16)[0])


def _cases(fmt: str, seed: int) -> np.ndarray:
    """fp64 test values around the representable points of fmt."""
    rng = np.random.default_rng(seed)
    if fmt == "bf16":
        b = rng.integers(0x0001, 0x7F7F, 3000).astype(np.uint32)
        lo = (b << 16).view(np.float32).astype(np.float64)
        hi = ((b + 1) << 16).view(np.float32).astype(np.float64)
    else:
        b = rng.integers(0x0001, 0x7BFF, 3000).astype(np.uint16)
        lo = b.view(np.float16).astype(np.float64)
        hi = (b + 1).astype(np.uint16).view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2                              # exact in fp64: a tie of either parity
    vals = [mid, np.nextafter(mid, np.inf), np.nextafter(mid, -np.inf), lo, hi,
            mid * (1 + 2.0 ** -40), mid * (1 - 2.0 ** -40),    # fp32 would round these onto the tie
            lo + (hi - lo) * rng.random(lo.size)]
    v = np.concatenate(vals)
    v = np.concatenate([v, -v])
    return v


def test_f64_to_bf16_bits_exact_rounding():
    Y = _cases("bf16", 1)
    got = C.f64_to_bf16_bits(Y)
    for y, g in zip(Y.tolist(), got.tolist()):
        ref = _rne_fraction(y, 8, -126)
        assert g == _bf16_bits_of(ref, y), (y, hex(g))


def test_f64_to_f16_bits_exact_rounding():
    Y = _cases("fp16", 2)
    sub = np.array([2.0 ** -24 * (k + 0.5) for k in range(0, 40)] + [2.0 ** -14 * 0.75, 2.0 ** -15 * 1.5])
    Y = np.concatenate([Y, sub, -sub])
    got = C.f64_to_f16_bits(Y)
    for y, g in zip(Y.tolist(), got.tolist()):
        ref = _rne_fraction(y, 11, -14)
        assert g == _f16_bits_of(ref, y), (y, hex(g))


def test_oracle_f32_to_f16_rne_exact_rounding():
    Y = _cases("fp16", 3).astype(np.float32)          # fp32 inputs: ties stay exact in fp32
    got = O.f32_to_f16_rne(Y)
    for y, g in zip(Y.astype(np.float64).tolist(), got.tolist()):
        assert g == _f16_bits_of(_rne_fraction(y, 11, -14), y), (y, hex(g))


def test_check_half_strict_rejects_two_ulps():
    Y = np.array([1.0 + 2.0 ** -7 * 0.25, 3.0])
    ref = C.f64_to_bf16_bits(Y)
    two_off = (ref.astype(np.int64) + 2).astype(np.uint16)
    T = np.abs(Y) * 1e6                               # a huge T would rescue the loose form
    C.check_half(two_off, Y, T, "bf16")               # loose: passes through the T escape
    try:
        C.check_half(two_off, Y, T, "bf16", strict=True)
    except AssertionError:
        pass
    else:
        raise AssertionError("strict check accepted a 2-ulp error")
    C.check_half((ref.astype(np.int64) + 1).astype(np.uint16), Y, T, "bf16", strict=True)
