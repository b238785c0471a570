"""Pins of the oracle's scalar building blocks against things other than itself:
library routines (numpy's IEEE binary16 conversion), exact rational arithmetic
(fractions.Fraction), and Philox-4x32-10 against cuRAND's implementation.
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
# Philox-4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11) pinned to an independent
# implementation: cuRAND's host generator CURAND_RNG_PSEUDO_PHILOX4_32_10
# (NVIDIA's CUDA library, run on the CPU).  With seed s it emits block m
# (4 words) = Philox(counter = (x, y, z, 0), key = (s mod 2^32, s >> 32))
# where m = (y * 2^32 + x) * 65536 + z: 65,536 interleaved subsequences.  A
# generator offset of 4m starts the stream at block m, which reaches the
# first three counter words; the fourth is pinned on the GPU
# (tests/test_gpu_philox.py, cuRAND's device API).
_CURAND = None


def _curand():
    global _CURAND
    if _CURAND is None:
        import ctypes
        import glob
        import os
        import torch
        paths = glob.glob(os.path.join(os.path.dirname(torch.__file__), "..", "nvidia", "curand", "lib",
                                       "libcurand.so*")) + glob.glob("/usr/local/cuda/lib64/libcurand.so*")
        for path in paths:
            try:
                _CURAND = ctypes.CDLL(path)
                break
            except OSError:
                continue
        if _CURAND is None:
            pytest.skip("libcurand not found")
    return _CURAND


def _curand_block(seed, x, y, z):
    import ctypes
    lib = _curand()
    gen = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), 161) == 0   # PHILOX4_32_10
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        block = ((y << 32) + x) * 65536 + z
        assert lib.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(4 * block)) == 0
        out = (ctypes.c_uint32 * 4)()
        assert lib.curandGenerate(gen, out, ctypes.c_size_t(4)) == 0
        return tuple(int(v) for v in out)
    finally:
        lib.curandDestroyGenerator(gen)


def test_philox_matches_curand():
    rng = np.random.default_rng(20260511)
    for _ in range(48):
        seed = int(rng.integers(0, 2**63)) * 2 + int(rng.integers(0, 2))
        x = int(rng.integers(0, 2**32))
        y = int(rng.integers(0, 2**13))
        z = int(rng.integers(0, 65536))
        key = np.array([seed & 0xFFFFFFFF, seed >> 32], np.uint32)
        got = tuple(int(v) for v in O.philox4x32_10(np.array([x, y, z, 0], np.uint32), key))
        assert got == _curand_block(seed, x, y, z), (seed, x, y, z)


def test_philox_edges_match_curand():
    for seed in (0, 2**64 - 1):
        for x, y, z in ((0, 0, 0), (2**32 - 1, 0, 65535), (1, 1, 1)):
            key = np.array([seed & 0xFFFFFFFF, seed >> 32], np.uint32)
            got = tuple(int(v) for v in O.philox4x32_10(np.array([x, y, z, 0], np.uint32), key))
            assert got == _curand_block(seed, x, y, z)


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
