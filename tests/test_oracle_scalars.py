"""Pins of the oracle's scalar building blocks against things other than itself:
library routines (numpy's IEEE binary16 conversion), exact rational arithmetic
(fractions.Fraction), and the published known-answer vectors of Philox-4x32-10.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle as O


# ---------------------------------------------------------------- fp16 ----

def _numpy_f16_bits(x):
    with np.errstate(over="ignore"):
        return np.asarray(x, np.float32).astype(np.float16).view(np.uint16)


def test_f32_to_f16_matches_numpy_on_random_bit_patterns():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2**32, size=1 << 21, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    finite = np.isfinite(x)
    got = O.f32_to_f16_rn(x[finite])
    np.testing.assert_array_equal(got, _numpy_f16_bits(x[finite]))


def test_f32_to_f16_matches_numpy_near_the_half_range():
    # every float32 whose exponent lies in the binary16 range or just around it,
    # sampled densely around the rounding midpoints
    rng = np.random.default_rng(2)
    e = rng.integers(-27, 17, size=1 << 20)
    m = rng.integers(0, 1 << 23, size=1 << 20)
    # put a fraction of the samples exactly on or next to a binary16 midpoint
    m[: 1 << 18] = (m[: 1 << 18] & ~0x1FFF) | 0x1000
    m[1 << 18: 1 << 19] = (m[1 << 18: 1 << 19] & ~0x1FFF) | 0x0FFF
    bits = (((e + 127) << 23) | m).astype(np.uint32)
    sign = rng.integers(0, 2, size=bits.size).astype(np.uint32) << 31
    x = (bits | sign).view(np.float32)
    np.testing.assert_array_equal(O.f32_to_f16_rn(x), _numpy_f16_bits(x))


def test_f32_to_f16_special_values():
    specials = np.array([0.0, -0.0, np.inf, -np.inf, 65504.0, 65519.996, 65520.0, 1e30,
                         2.0**-24, 2.0**-25, 2.0**-25 * 1.0000001, 2.0**-14, 2.0**-14 * (1 - 2.0**-12)],
                        np.float32)
    np.testing.assert_array_equal(O.f32_to_f16_rn(specials), _numpy_f16_bits(specials))
    assert (O.f32_to_f16_rn(np.array([np.nan], np.float32))[0] & 0x7C00) == 0x7C00


def test_f16_to_f32_exhaustive():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = O.f16_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    np.testing.assert_array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    assert np.isnan(got[nan]).all()


# ------------------------------------------------------ division toward zero

@pytest.mark.parametrize("qmax", [3, 7, 31, 127])
def test_div_rz_is_the_largest_float_not_above_the_quotient(qmax):
    rng = np.random.default_rng(qmax)
    m = np.exp(rng.normal(0, 8, size=4000)).astype(np.float32)
    m = m[(m > 0) & np.isfinite(m)]
    a = np.full(m.shape, qmax, np.float32)
    got = O.div_rz(a, m)
    for q, mm in zip(got.tolist(), m.tolist()):
        qf, mf = Fraction(q), Fraction(mm)
        assert qf * mf <= qmax
        up = Fraction(float(np.nextafter(np.float32(q), np.float32(np.inf))))
        assert up * mf > qmax


def test_div_rz_exact_quotients_are_kept():
    m = np.array([1.0, 0.5, 127.0, 2.0**-20, 3.0], np.float32)
    a = np.array([127.0, 127.0, 127.0, 127.0, 6.0], np.float32)
    np.testing.assert_array_equal(O.div_rz(a, m), (a.astype(np.float64) / m).astype(np.float32))


# --------------------------------------------------------------- Philox ----
# Known-answer vectors published with the Random123 library (Salmon et al.,
# SC'11), file kat_vectors, generator philox4x32 with 10 rounds.
PHILOX_KAT = [
    ((0x00000000, 0x00000000, 0x00000000, 0x00000000), (0x00000000, 0x00000000),
     (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
    ((0xffffffff, 0xffffffff, 0xffffffff, 0xffffffff), (0xffffffff, 0xffffffff),
     (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
    ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
     (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1)),
]


@pytest.mark.parametrize("ctr,key,expect", PHILOX_KAT)
def test_philox_known_answers(ctr, key, expect):
    assert tuple(int(x) for x in O.philox4x32_10(ctr, key)) == expect


# ------------------------------------------------- stochastic-rounding offsets

def test_sr_delta_grid_and_range():
    vals = np.array([O.sr_delta(123, 5, 7, 3, s, j) for s in range(8) for j in range(128)])
    scaled = vals * 2.0**17
    assert np.all(np.abs(vals) < 0.5)
    assert np.all(scaled == np.round(scaled))              # multiples of 2^-17
    assert np.all(np.mod(np.round(scaled), 2) == 1)        # odd multiples: never 0, symmetric
    assert abs(vals.mean()) < 4 * 0.29 / np.sqrt(vals.size)


def test_sr_delta_is_a_pure_function_of_its_counter():
    a = [O.sr_delta(9, 1, 2, 3, s, j) for s in range(4) for j in range(8)]
    b = [O.sr_delta(9, 1, 2, 3, s, j) for s in range(4) for j in range(8)]
    assert a == b
    c = [O.sr_delta(9, 2, 2, 3, s, j) for s in range(4) for j in range(8)]
    assert a != c
    # the two columns of one 32-bit word come from its high and low halves
    ctr = np.array([0, 1, 2, 3], np.uint32)
    out = O.philox4x32_10(ctr, np.array([9, 0], np.uint32))
    w = int(out[0])
    assert O.sr_delta(9, 1, 2, 3, 0, 0) == (2 * (w >> 16) - 65535) * 2.0**-17
    assert O.sr_delta(9, 1, 2, 3, 0, 1) == (2 * (w & 0xFFFF) - 65535) * 2.0**-17
