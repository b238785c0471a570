"""Pins of the oracle's scalar building blocks against things other than itself:
library routines (numpy's IEEE binary16 conversion), exact rational arithmetic
(fractions.Fraction), and the pcg4d hash by its inverse and its statistics.
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


# ---------------------------------------------------------------- pcg4d ----
# pcg4d (Jarzynski and Olano, "Hash Functions for GPU Rendering", JCGT 2020):
# the pins check what the stochastic rounding needs of it, each of which a
# plausible slip (a dropped mixing step, a wrong shift, a swapped word)
# breaks: every step is invertible, so the map is a bijection (the inverse,
# written out here, recovers random inputs); the 16-bit halves the rounding
# uses are uniform over consecutive counters (chi-square); neighbouring
# counters give unrelated words (correlation of halves, and about half of the
# output bits flip when one input bit flips).
def _pcg4d_inverse(o):
    x, y, z, w = (int(v) for v in o)
    M = 0xFFFFFFFF
    w = (w - y * z) & M
    z = (z - x * y) & M
    y = (y - z * x) & M
    x = (x - y * w) & M

    def unshift(v):
        return v ^ (v >> 16)            # a 16-bit xorshift of a 32-bit word is its own inverse
    x, y, z, w = unshift(x), unshift(y), unshift(z), unshift(w)
    w = (w - y * z) & M
    z = (z - x * y) & M
    y = (y - z * x) & M
    x = (x - y * w) & M
    ainv = pow(1664525, -1, 2**32)
    return [((v - 1013904223) * ainv) & M for v in (x, y, z, w)]


def test_pcg4d_is_a_bijection():
    rng = np.random.default_rng(5)
    for _ in range(200):
        v = rng.integers(0, 2**32, 4, dtype=np.uint64).astype(np.uint32)
        assert _pcg4d_inverse(O.pcg4d(v)) == [int(x) for x in v]


def _halves(n, step=3, b=7, h=2):
    out = np.array([O.pcg4d(np.array([i, step, b, h], np.uint32)) for i in range(n)], np.uint64)
    return np.concatenate([out >> 16, out & 0xFFFF]).ravel()


def test_pcg4d_halves_are_uniform():
    x = _halves(8192)                                   # 65,536 16-bit values
    counts = np.bincount((x >> 10).astype(np.int64), minlength=64)   # 64 bins
    expect = x.size / 64
    chi2 = float(((counts - expect) ** 2 / expect).sum())
    assert chi2 < 120, chi2                             # 63 dof: p < 1e-5 above 120


def test_pcg4d_neighbouring_counters_are_unrelated():
    n = 8192
    out = np.array([O.pcg4d(np.array([i, 1, 0, 0], np.uint32)) for i in range(n)], np.uint64)
    a = (out[:-1, 0] >> 16).astype(np.float64)
    b = (out[1:, 0] >> 16).astype(np.float64)
    assert abs(np.corrcoef(a, b)[0, 1]) < 4 / np.sqrt(n)
    # avalanche: one flipped input bit flips about half of the 128 output bits
    rng = np.random.default_rng(8)
    flips = []
    for _ in range(400):
        v = rng.integers(0, 2**32, 4, dtype=np.uint64).astype(np.uint32)
        bit = int(rng.integers(0, 128))
        u = v.copy()
        u[bit // 32] ^= np.uint32(1 << (bit % 32))
        d = O.pcg4d(v) ^ O.pcg4d(u)
        flips.append(sum(bin(int(t)).count("1") for t in d))
    assert 56 < np.mean(flips) < 72, np.mean(flips)


# ------------------------------------------------- stochastic-rounding offsets

def test_sr_offset_grid_and_range():
    vals = np.array([O.sr_offset(123, 5, 7, 3, s, j) for s in range(8) for j in range(128)])
    scaled = vals * 2.0**16
    assert np.all((vals >= 0.0) & (vals < 1.0))
    assert np.all(scaled == np.round(scaled))              # multiples of 2^-16
    # uniform on the grid: mean (1 - 2^-16) / 2, variance ~ 1/12
    assert abs(vals.mean() - (0.5 - 2.0**-17)) < 4 * 0.29 / np.sqrt(vals.size)
    assert abs(vals.var() - 1.0 / 12) < 0.01
    counts = np.histogram(vals, bins=8, range=(0.0, 1.0))[0]
    exp = vals.size / 8
    assert np.sum((counts - exp) ** 2 / exp) < 24.3        # chi-square, 7 dof, p ~ 0.001


def test_sr_offset_is_a_pure_function_of_its_counter():
    a = [O.sr_offset(9, 1, 2, 3, s, j) for s in range(4) for j in range(8)]
    b = [O.sr_offset(9, 1, 2, 3, s, j) for s in range(4) for j in range(8)]
    assert a == b
    c = [O.sr_offset(9, 2, 2, 3, s, j) for s in range(4) for j in range(8)]
    assert a != c
    # the two columns of one 32-bit word come from its high and low halves;
    # the input is (tile, step, request ^ low seed word, head ^ high seed word)
    out = O.pcg4d(np.array([0, 1, 2 ^ 9, 3], np.uint32))
    w = int(out[0])
    assert O.sr_offset(9, 1, 2, 3, 0, 0) == (w >> 16) * 2.0**-16
    assert O.sr_offset(9, 1, 2, 3, 0, 1) == (w & 0xFFFF) * 2.0**-16
