"""Pins of the oracle's bf16 rounding helpers (CPU only).

Every bit-exact dequantisation claim and every bf16 rounding point of the layer
oracle rests on ``oracle.bf16``.  These pins check it against conversions that
share nothing with it:

* fp32 -> bf16: torch's own ``Tensor.to(torch.bfloat16)`` (round to nearest, ties
  to even), on random values over the whole exponent range and on constructed bit
  patterns: exact ties with the kept bit even and odd, one ulp either side of a
  tie, negatives, fp32 subnormals, values next to the bf16 maximum;
* float64 -> bf16 in one rounding: exact rational arithmetic with
  ``fractions.Fraction``, whose ``round`` goes to the nearest integer with ties to
  even.  torch cannot serve here: it converts float64 through fp32 first and so
  rounds twice (1 + 2^-8 + 2^-30 becomes 1, not 1 + 2^-7).  The domain of
  ``round_f64`` is the normal bf16 range, |x| in [2^-126, bf16 max]; below it the
  helper keeps 8 significant bits instead of the subnormal grid, which no tensor
  of this workload reaches.
"""
from fractions import Fraction

import numpy as np
import torch

from oracle import bf16


def _torch_bits(x32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _f32(bits) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint32).view(np.float32)


def _special_f32_patterns() -> np.ndarray:
    pats = []
    rng = np.random.default_rng(11)
    hi = rng.integers(0, 1 << 15, 400, dtype=np.uint32) << 16          # sign + exponent + 7 kept bits
    for low in (0x8000, 0x7FFF, 0x8001, 0x0000, 0xFFFF, 0x0001):
        pats.append(hi | np.uint32(low))
    # exact ties with the kept lsb even and odd, both signs
    for kept in (0x3F80, 0x3F81, 0x4000, 0x4001, 0xBF80, 0xBF81):
        pats.append(np.array([(kept << 16) | 0x8000], np.uint32))
    # fp32 subnormals (exponent field 0), including ties and the largest one
    sub = np.array([0x00000001, 0x00008000, 0x00018000, 0x00017FFF, 0x007FFFFF, 0x00400000,
                    0x80008000, 0x80018000, 0x807FFFFF], np.uint32)
    pats.append(sub)
    # next to the bf16 maximum (0x7F7F): below, at, and the tie that rounds up to infinity
    near_max = np.array([0x7F7E8000, 0x7F7F0000, 0x7F7F7FFF, 0x7F7F8000, 0x7F7E7FFF, 0xFF7F7FFF, 0xFF7F8000],
                        np.uint32)
    pats.append(near_max)
    pats.append(np.array([0x00000000, 0x80000000, 0x3F800000, 0xBF800000], np.uint32))
    return np.concatenate(pats)


def test_f32_to_bf16_bits_matches_torch_on_constructed_patterns():
    x = _f32(_special_f32_patterns())
    x = x[np.isfinite(x)]
    np.testing.assert_array_equal(bf16.f32_to_bf16_bits(x), _torch_bits(x))


def test_f32_to_bf16_bits_matches_torch_over_the_exponent_range():
    rng = np.random.default_rng(12)
    mant = rng.normal(0, 1, 200_000)
    expo = rng.integers(-140, 127, mant.size)
    x = (mant * np.exp2(expo.astype(np.float64))).astype(np.float32)
    x = x[np.isfinite(x)]
    np.testing.assert_array_equal(bf16.f32_to_bf16_bits(x), _torch_bits(x))
    np.testing.assert_array_equal(bf16.round_f32(x), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_f32_to_bf16_ties_go_to_even():
    # 1 + 2^-8 lies halfway between bf16 1 and 1 + 2^-7: the even neighbour 1 wins;
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even): up.
    x = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), -(1 + 3 * 2.0 ** -8)], np.float32)
    np.testing.assert_array_equal(bf16.round_f32(x).astype(np.float64),
                                  [1.0, 1 + 2.0 ** -6, -1.0, -(1 + 2.0 ** -6)])


def _rne_fraction(x: float) -> float:
    """x rounded to 8 significant bits, ties to even, in exact arithmetic."""
    if x == 0.0:
        return x
    f = Fraction(x)
    a = abs(f)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    q = Fraction(2) ** (e - 7)                      # ulp of an 8-bit significand at 2^e
    r = round(f / q) * q                            # Fraction.__round__: half to even
    return float(r)


def test_round_f64_matches_exact_rounding():
    rng = np.random.default_rng(13)
    mant = rng.normal(0, 1, 20_000)
    expo = rng.integers(-120, 120, mant.size)
    x = mant * np.exp2(expo.astype(np.float64))
    got = bf16.round_f64(x)
    ref = np.array([_rne_fraction(float(v)) for v in x])
    np.testing.assert_array_equal(got, ref)


def test_round_f64_ties_and_near_ties():
    vals = []
    for e in (-100, -7, 0, 5, 100):
        for k in (128, 129, 200, 255):              # kept 8-bit significands, even and odd
            base = k * 2.0 ** (e - 7)
            half = 2.0 ** (e - 8)
            tiny = half * 2.0 ** -40
            for s in (1.0, -1.0):
                vals += [s * (base + half), s * (base + half + tiny), s * (base + half - tiny), s * base]
    x = np.array(vals)
    got = bf16.round_f64(x)
    ref = np.array([_rne_fraction(float(v)) for v in x])
    np.testing.assert_array_equal(got, ref)
    # spelled out: halfway above an even significand stays, above an odd one goes up
    assert bf16.round_f64(np.array([1 + 2.0 ** -8]))[0] == 1.0
    assert bf16.round_f64(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6
    assert bf16.round_f64(np.array([1 + 2.0 ** -8 + 2.0 ** -30]))[0] == 1 + 2.0 ** -7


def test_round_f64_agrees_with_fp32_path_on_fp32_values():
    # on values that are already fp32 the one rounding from float64 and the fp32 path agree
    rng = np.random.default_rng(14)
    x = (rng.normal(0, 1, 50_000) * np.exp2(rng.integers(-100, 100, 50_000))).astype(np.float32)
    np.testing.assert_array_equal(bf16.round_f64(x.astype(np.float64)), bf16.round_f32(x).astype(np.float64))
