"""Pins of the oracle's calibration, quantizer and dequantizer.

* brute force at d_k = d_v = 4: every code is the nearest point of the row's
  grid {z r : |z| <= qmax} (exhaustive search, exact rationals);
* the absmax element of a row maps to +-qmax; zero rows and columns;
* values already on the grid round-trip exactly (an invariant of the method);
* reconstruction error within half a grid step;
* the precision map on states whose ranking is known by construction.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from linear_attention_recurrent_delta_b200 import workloads as W

D4_GROUPS = [(1, "int", 8), (2, "int", 6), (1, "int", 4)]


def _nearest_on_grid(t, r, qmax):
    """argmin_z |t - z r| over z in [-qmax, qmax], ties to the even z (exact)."""
    tf, rf = Fraction(t), Fraction(r)
    best = None
    for z in range(-qmax, qmax + 1):
        d = abs(tf - z * rf)
        if best is None or d < best[0] or (d == best[0] and z % 2 == 0):
            best = (d, z)
    return best[1]


@pytest.mark.parametrize("col_scales", [False, True])
@pytest.mark.parametrize("seed", range(6))
def test_quantizer_brute_force_d4(col_scales, seed):
    rng = np.random.default_rng(100 + seed)
    fmt = O.make_format(D4_GROUPS, d_k=4, d_v=4, col_scales=col_scales)
    S = (rng.normal(size=(4, 4)) * np.exp(rng.normal(size=(4, 1))) * np.exp(rng.normal(size=(1, 4))))
    S = S.astype(np.float32)
    perm = rng.permutation(4).astype(np.int32)
    page = O.quantize_page(fmt, S, perm)
    absS = np.abs(S).astype(np.float64)
    for j in range(4):
        expect_c = absS[:, j].max() if col_scales else 1.0
        assert page.c[j] == np.float32(expect_c)
    band = 0
    for s in range(4):
        qmax = O.row_qmax(fmt, s)
        T = S[perm[s]] * (np.float32(1) / page.c) if col_scales else S[perm[s]]
        T = T.astype(np.float32)
        m = np.abs(T).max()
        assert page.r[s] == np.float32(m / np.float32(qmax))
        # the absmax element lands on +-qmax
        jm = int(np.argmax(np.abs(T)))
        assert abs(page.code[s, jm]) == qmax
        for j in range(4):
            z = _nearest_on_grid(float(T[j]), float(m) / qmax, qmax)
            x = Fraction(float(T[j])) * qmax / Fraction(float(m))
            if abs(x - (x.numerator // x.denominator) - Fraction(1, 2)) < Fraction(1, 10**5):
                band += 1
                continue
            assert page.code[s, j] == z, (s, j)
    assert band == 0


@pytest.mark.parametrize("name", ["stepquant6", "int8row", "stepquant4_kda", "damp"])
def test_quantizer_error_bound_and_dequantizer(name):
    w = [x for x in W.WORKLOADS if x.fmt == name][0]
    fmt = O.format_from_spec(W.FORMATS[name])
    S = W.initial_state(w, batch=2)[:, :2].numpy()
    perm = O.rank_rows(fmt, S)
    for b in range(2):
        for h in range(2):
            page = O.quantize_page(fmt, S[b, h], perm[h])
            Sh = O.dequantize_page(fmt, page, perm[h]).astype(np.float64)
            err = np.abs(Sh - S[b, h])
            for s in range(128):
                kap = perm[h][s]
                if O.row_qmax(fmt, s):
                    bound = 0.5 * page.r[s] * page.c.astype(np.float64) * (1 + 1e-5) + 1e-6 * np.abs(S[b, h, kap])
                else:  # FP16 rows: half an fp16 spacing, relative
                    bound = 2.0**-11 * np.abs(S[b, h, kap]) * page.c + 2.0**-25 * page.c
                assert np.all(err[kap] <= bound), (name, s)


@pytest.mark.parametrize("name", ["int8row", "damp"])
def test_values_on_the_grid_round_trip_exactly(name):
    """Values already on the grid round-trip exactly through
    quantize/dequantize (per-row formats; power-of-two row scales)."""
    fmt = O.format_from_spec(W.FORMATS[name])
    rng = np.random.default_rng(5)
    perm = rng.permutation(128).astype(np.int32)
    S = np.zeros((128, 128), np.float32)
    for s in range(128):
        kap = perm[s]
        qmax = O.row_qmax(fmt, s)
        if qmax:
            z = rng.integers(-qmax, qmax + 1, 128)
            z[rng.integers(128)] = qmax * rng.choice([-1, 1])
            S[kap] = z * np.float32(2.0 ** rng.integers(-20, 10))
        else:
            S[kap] = rng.integers(-2048, 2049, 128) * np.float32(2.0 ** rng.integers(-20, 4))
    page = O.quantize_page(fmt, S, perm)
    np.testing.assert_array_equal(O.dequantize_page(fmt, page, perm), S)


def test_zero_rows_and_columns():
    fmt = O.format_from_spec(W.FORMATS["stepquant6"])
    S = np.random.default_rng(3).normal(size=(128, 128)).astype(np.float32)
    S[5] = 0
    S[:, 7] = 0
    perm = np.arange(128, dtype=np.int32)
    page = O.quantize_page(fmt, S, perm)
    assert page.c[7] == 1.0
    assert page.r[5] == 0.0 and np.all(page.code[5] == 0)
    assert np.all(page.code[:, 7] == 0)
    np.testing.assert_array_equal(O.dequantize_page(fmt, page, perm)[5], 0)


def test_rank_rows_known_ranking():
    fmt = O.make_format(D4_GROUPS, d_k=4, d_v=4)
    base = np.random.default_rng(0).normal(size=(3, 2, 4, 4)).astype(np.float32)
    scale = np.array([1.0, 10.0, 0.1, 5.0], np.float32)
    S = base / np.sqrt((base**2).sum(axis=(0, 3), keepdims=True)) * scale[None, None, :, None]
    perm = O.rank_rows(fmt, S)
    # ranking 1 > 3 > 0 > 2: group sizes 1, 2, 1; ascending key channel inside a group
    np.testing.assert_array_equal(perm, [[1, 0, 3, 2], [1, 0, 3, 2]])
    # a retention weight reorders head 1: row 2 weighted by 1000 scores 10,
    # between row 3 (25) and row 0 (1): ranking 1 > 3 > 2 > 0
    wgt = np.ones((2, 4), np.float32)
    wgt[1, 2] = 1000
    perm = O.rank_rows(fmt, S, wgt)
    np.testing.assert_array_equal(perm, [[1, 0, 3, 2], [1, 2, 3, 0]])


def test_rank_rows_ties_prefer_lower_channels():
    fmt = O.make_format(D4_GROUPS, d_k=4, d_v=4)
    S = np.zeros((1, 1, 4, 4), np.float32)
    np.testing.assert_array_equal(O.rank_rows(fmt, S), [[0, 1, 2, 3]])
    S[0, 0, 3] = 1
    np.testing.assert_array_equal(O.rank_rows(fmt, S), [[3, 0, 1, 2]])


def test_rank_rows_is_a_permutation_into_groups():
    fmt = O.format_from_spec(W.FORMATS["stepquant4_kda"])
    S = W.initial_state(W.WORKLOADS[3], batch=3)[:, :3].numpy()
    perm = O.rank_rows(fmt, S)
    score = (S.astype(np.float64) ** 2).sum(axis=(0, 3))
    for h in range(3):
        assert sorted(perm[h]) == list(range(128))
        start = 0
        prev_min = np.inf
        for rows, _, _ in W.FORMATS["stepquant4_kda"]["groups"]:
            grp = perm[h][start:start + rows]
            assert list(grp) == sorted(grp)
            # every row of an earlier group outscores every row of a later one
            assert score[h, grp].max() <= prev_min
            prev_min = score[h, grp].min()
            start += rows
