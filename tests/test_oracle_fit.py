"""Pins of the joint fit of row and column scales (orc_quantize_page_fit).

STEPQuant fits key-row and value-column scales jointly from the state and
each key row's impact on the output (paper-cards page, STEPQuant abstract).
The oracle minimizes the impact-weighted squared reconstruction error by
alternating exact steps from the absmax scales.  Pinned here:

* no fitting (iters = 0) is the absmax quantizer, bit for bit;
* the objective never rises from round to round, and the final page's
  objective, recomputed here in exact rational arithmetic at 4 x 4, is the
  reported one;
* every final code is the nearest code (clamped) for the fitted scales,
  exhaustively checked in exact rationals at 4 x 4;
* first-order optimality of the last scale update: the row scales are least
  squares for the codes they were fitted to, so scaling one by (1 +- eps)
  raises the row's error; the same for an impact-weighted column scale;
* the fit improves on absmax on the workloads' states (strictly where there
  are column scales), and weighting one row heavily lowers that row's error
  compared with uniform weights.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from linear_attention_recurrent_delta_b200 import workloads as W

FORMATS_D4 = [
    ([(1, "int", 8), (2, "int", 3), (1, "int", 2)], True),
    ([(4, "int", 3)], True),
    ([(2, "int", 4), (2, "int", 2)], False),
]


def _objective_exact(fmt, S, perm, page, w=None):
    e = Fraction(0)
    for s in range(fmt.d_k):
        if O.row_kind(fmt, s) != 0:
            continue
        kap = perm[s]
        row = Fraction(0)
        for j in range(fmt.d_v):
            d = Fraction(float(S[kap, j])) - int(page.code[s, j]) * Fraction(float(page.r[s])) * \
                Fraction(float(page.c[j]))
            row += d * d
        e += (Fraction(float(w[kap])) if w is not None else 1) * row
    return e


def _case4(groups, col, seed):
    rng = np.random.default_rng(seed)
    fmt = O.make_format(groups, d_k=4, d_v=4, col_scales=col)
    S = (rng.standard_normal((4, 4)) * np.exp(rng.standard_normal((4, 1))) *
         np.exp(rng.standard_normal((1, 4)))).astype(np.float32)
    perm = rng.permutation(4).astype(np.int32)
    w = (rng.random(4) + 0.1).astype(np.float32)
    return fmt, S, perm, w


@pytest.mark.parametrize("groups,col", FORMATS_D4)
def test_no_fit_is_the_absmax_quantizer(groups, col):
    fmt, S, perm, w = _case4(groups, col, 1)
    a = O.quantize_page(fmt, S, perm)
    b, _ = O.quantize_page_fit(fmt, S, perm, w, iters=0)
    assert np.array_equal(a.code, b.code)
    assert np.array_equal(a.r.view(np.uint32), b.r.view(np.uint32))
    assert np.array_equal(a.c.view(np.uint32), b.c.view(np.uint32))


@pytest.mark.parametrize("groups,col", FORMATS_D4)
@pytest.mark.parametrize("seed", range(5))
def test_brute_force_d4(groups, col, seed):
    fmt, S, perm, w = _case4(groups, col, 10 + seed)
    page, err = O.quantize_page_fit(fmt, S, perm, w, iters=5)
    # monotone, and the reported final objective is the page's
    assert np.all(np.diff(err) <= 1e-12 * err[0]), err
    exact = _objective_exact(fmt, S, perm, page, w)
    assert abs(float(exact) - err[-1]) <= 1e-12 * max(err[-1], 1e-300)
    # every code the nearest (clamped) code for the fitted scales, in exact rationals
    for s in range(4):
        qmax = O.row_qmax(fmt, s)
        r = Fraction(float(page.r[s]))
        for j in range(4):
            d = r * Fraction(float(page.c[j]))
            z = int(page.code[s, j])
            assert -qmax <= z <= qmax
            if d == 0:
                assert z == 0
                continue
            x = Fraction(float(S[perm[s], j])) / d
            for cand in range(-qmax, qmax + 1):
                assert abs(x - z) <= abs(x - cand), (s, j, z, cand)


def _row_err(S_row, z, r, c):
    d = S_row.astype(np.float64) - z.astype(np.float64) * float(r) * c.astype(np.float64)
    return float(d @ d)


@pytest.mark.parametrize("name", ["stepquant6", "stepquant4_kda"])
def test_last_updates_are_least_squares(name):
    """Fitted once (iters = 1), the page's codes are the nearest codes for the
    fitted scales, which may differ from the codes the scales were fitted to;
    so the optimality check refits with those first codes: iters = 1 scales
    are least squares for the iters = 1 starting codes (the absmax codes,
    re-derived by the division rule)."""
    w = [x for x in W.WORKLOADS if x.fmt == name][0]
    fmt = O.format_from_spec(w.format)
    S = W.initial_state(w, batch=1).numpy()
    perm = O.rank_rows(fmt, S)[0]
    S = S[0, 0]
    imp = (np.random.default_rng(3).random(128) + 0.5).astype(np.float32)
    base = O.quantize_page(fmt, S, perm)
    page, _ = O.quantize_page_fit(fmt, S, perm, imp, iters=1)
    # the codes the round fitted to: nearest codes for the absmax scales
    z0 = np.zeros((128, 128), np.int64)
    for s in range(128):
        qmax = O.row_qmax(fmt, s)
        d = base.r[s].astype(np.float64) * base.c.astype(np.float64)
        z0[s] = np.clip(np.rint(S[perm[s]].astype(np.float64) / d), -qmax, qmax)
    for s in (0, 40, 100, 127):
        e0 = _row_err(S[perm[s]], z0[s], page.r[s], base.c)
        for eps in (1e-4, -1e-4):
            assert _row_err(S[perm[s]], z0[s], page.r[s] * (1 + eps), base.c) >= e0
    # the column update used the new row scales and the same codes
    zr = z0 * page.r.astype(np.float64)[:, None]
    Snat = S[perm].astype(np.float64)
    wk = imp[perm].astype(np.float64)
    for j in (0, 63, 127):
        def col_err(cj):
            d = Snat[:, j] - zr[:, j] * cj
            return float(wk @ (d * d))
        e0 = col_err(float(page.c[j]))
        for eps in (1e-4, -1e-4):
            assert col_err(float(page.c[j]) * (1 + eps)) >= e0


@pytest.mark.parametrize("name", list(W.FORMATS))
def test_fit_improves_on_absmax(name):
    w = [x for x in W.WORKLOADS if x.fmt == name][0]
    fmt = O.format_from_spec(w.format)
    S = W.initial_state(w, batch=1).numpy()
    perm = O.rank_rows(fmt, S)
    for h in range(3):
        _, err = O.quantize_page_fit(fmt, S[0, h], perm[h], None, iters=4)
        assert np.all(np.diff(err) <= 1e-12 * err[0])
        if fmt.col_scales:
            assert err[-1] < 0.9 * err[0], (h, err)
        else:
            assert err[-1] <= err[0]


def test_heavy_impact_weight_lowers_that_rows_error():
    w = [x for x in W.WORKLOADS if x.fmt == "stepquant4_kda"][0]
    fmt = O.format_from_spec(w.format)
    S_all = W.initial_state(w, batch=1).numpy()
    perm = O.rank_rows(fmt, S_all)[0]
    S = S_all[0, 0]
    s = 100                                   # an INT3 row
    kap = perm[s]
    uni, _ = O.quantize_page_fit(fmt, S, perm, None, iters=4)
    heavy = np.ones(128, np.float32)
    heavy[kap] = 1e4
    wpg, _ = O.quantize_page_fit(fmt, S, perm, heavy, iters=4)
    e_uni = _row_err(S[kap], uni.code[s], uni.r[s], uni.c)
    e_w = _row_err(S[kap], wpg.code[s], wpg.r[s], wpg.c)
    assert e_w < e_uni, (e_w, e_uni)
