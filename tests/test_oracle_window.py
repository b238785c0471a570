"""Pins of the oracle's per-window decode step (orc_window_step_f32).

Within a window the packed page stays fixed and the step's high-precision
updates sit in a buffer; the state is requantized once, at the window's last
step.  Inside a window nothing is rounded to the quantized grid, so every
output of the window must be the exact gated delta rule run in fp64 from the
dequantized page, up to fp32 rounding.  The pins:

* o, the buffer's deltas D and its decayed keys K at every step against the
  fp64 matrix form S <- diag(a) S + beta k (v - (diag(a) S)^T k)^T from the
  dequantized page, every format, windows of 1 to 8 steps;
* the committed page against the fp64 state: each element within one
  quantization step of its new row scale (half a step for round to nearest);
  the cumulative decay P is reset to one; a second window started from the
  committed page again follows the fp64 rule from that page;
* brute force at d_k = d_v = 4 (one lane in the buffer dot products);
* a window of one step is the plain step: same codes (away from rounding
  midpoints), same row scales and o to a few ulps;
* alpha = 1, beta = 0 over a whole window leaves the page bit for bit;
  alpha = 0 at a step empties everything before it.
"""
import numpy as np
import pytest

import oracle as O
from linear_attention_recurrent_delta_b200 import workloads as W


def _rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def _dequant64(fmt, page, perm):
    """Natural-order state q_ij * r_i * c_j in double (FP16 rows: h_ij * c_j)."""
    S = np.zeros((fmt.d_k, fmt.d_v))
    for s in range(fmt.d_k):
        kind = O.row_kind(fmt, s)
        if kind == 0:
            x = page.code[s].astype(np.float64) * float(page.r[s])
        elif kind == 1:
            x = O.f16_to_f32(page.code[s].astype(np.uint16)).astype(np.float64)
        else:
            x = page.code[s].astype(np.uint32).view(np.float32).astype(np.float64)
        S[perm[s]] = x * (page.c.astype(np.float64) if fmt.col_scales else 1.0)
    return S


def _colscale(fmt, page):
    return page.c.astype(np.float64) if fmt.col_scales else np.ones(fmt.d_v)


def _evolve64(S0, steps):
    """The gated delta rule in fp64: per step (o, D_tau in state units, S)."""
    S = S0.copy()
    out = []
    for q, k, v, alpha, beta in steps:
        a = np.atleast_1d(alpha).astype(np.float64)
        S = (a[:, None] if a.size > 1 else float(a[0])) * S
        k64 = k.astype(np.float64)
        e = v.astype(np.float64) - S.T @ k64
        S = S + float(beta) * np.outer(k64, e)
        out.append((S.T @ q.astype(np.float64), float(beta) * e, S.copy()))
    return out


def _workload(name):
    w = [x for x in W.WORKLOADS if x.fmt == name][0]
    fmt = O.format_from_spec(W.FORMATS[name])
    S = W.initial_state(w, batch=1)[:, :1].numpy()
    perm = O.rank_rows(fmt, S)[0]
    page = O.quantize_page(fmt, S[0, 0], perm)
    return w, fmt, perm, page


def _inputs(w, first, n):
    steps = []
    for i in range(n):
        x = W.step_inputs(w, first + i, batch=1)
        steps.append(tuple(x[nm][0, 0].numpy() for nm in ("q", "k", "v", "alpha")) + (float(x["beta"][0, 0]),))
    return steps


def _run_window(fmt, page, perm, steps, seed=0, step0=0, b=0, h=0, plain=False):
    """Run one window over steps (commit at the last); returns per-step (o, P, K, D) copies."""
    n = len(steps)
    P = np.ones(fmt.d_k, np.float32)
    K = np.zeros((n, fmt.d_k), np.float32)
    D = np.zeros((n, fmt.d_v), np.float32)
    rec = []
    for t, (q, k, v, alpha, beta) in enumerate(steps):
        o, _ = O.window_step_f32(fmt, page, perm, P, K, D, t, t == n - 1, q, k, v, alpha, beta, seed=seed,
                                 step=step0 + t, b=b, h=h, plain=plain)
        rec.append((o, P.copy(), K.copy(), D.copy()))
    return rec


def _cumdecay(steps, first, last, d_k):
    """prod of the gates of steps first..last (inclusive) per key channel, fp64."""
    p = np.ones(d_k)
    for i in range(first, last + 1):
        a = np.atleast_1d(steps[i][3]).astype(np.float64)
        p = p * (a if a.size > 1 else float(a[0]))
    return p


@pytest.mark.parametrize("plain", [False, True])
@pytest.mark.parametrize("name", list(W.FORMATS))
@pytest.mark.parametrize("n", [1, 4, 8])
def test_window_outputs_follow_the_f64_rule(name, n, plain):
    w, fmt, perm, page = _workload(name)
    steps = _inputs(w, 40, n)
    S0 = _dequant64(fmt, page, perm)
    c = _colscale(fmt, page)
    ref = _evolve64(S0, steps)
    rec = _run_window(fmt, page.copy(), perm, steps, plain=plain)
    for t in range(n):
        o, P, K, D = rec[t]
        o64, d64, _ = ref[t]
        assert _rel_l2(o, o64) <= 1e-5, (t, _rel_l2(o, o64))
        # deltas are kept in column-normalised units: D[t] c == beta (v - S^T k)
        assert _rel_l2(D[t] * c, d64) <= 1e-5, (t, _rel_l2(D[t] * c, d64))
        if t < n - 1:   # after a commit P is back at one (checked below)
            np.testing.assert_allclose(P, _cumdecay(steps, 0, t, fmt.d_k), rtol=1e-5)
        for tau in range(t + 1):
            expect = steps[tau][1].astype(np.float64) * _cumdecay(steps, tau + 1, t, fmt.d_k)
            np.testing.assert_allclose(K[tau], expect, rtol=1e-5, atol=1e-30)


def _check_commit(fmt, page, S_ref):
    """Each committed element within one quantization step of the fp64 state
    (half a step plus rounding for round to nearest); FP16 rows to half an fp16 ulp."""
    Sq = _dequant64(fmt, page, np.arange(fmt.d_k))          # stored order
    c = _colscale(fmt, page)
    for s in range(fmt.d_k):
        kind = O.row_kind(fmt, s)
        ref = S_ref[s]
        err = np.abs(Sq[s] - ref)
        if kind == 0:
            unit = float(page.r[s]) * c
            frac = 1.0 if fmt.stochastic else 0.5
            assert np.all(err <= (frac + 1e-3) * unit + 1e-6 * np.abs(ref)), (s, (err / unit).max())
            # the new row scale covers the row's absolute maximum exactly
            m = np.abs(ref / c).max()
            assert abs(float(page.r[s]) * O.row_qmax(fmt, s) - m) <= 1e-5 * m
        elif kind == 1:
            assert np.all(err <= (2.0**-11 + 1e-5) * np.abs(ref) + 2.0**-25 * c), s


@pytest.mark.parametrize("name", list(W.FORMATS))
def test_commit_requantizes_the_f64_state_and_restarts(name):
    w, fmt, perm, page = _workload(name)
    steps = _inputs(w, 70, 6)
    S0 = _dequant64(fmt, page, perm)
    ref = _evolve64(S0, steps[:3])
    pg = page.copy()
    rec = _run_window(fmt, pg, perm, steps[:3], seed=9)
    np.testing.assert_array_equal(rec[-1][1], np.ones(fmt.d_k, np.float32))     # P reset
    _check_commit(fmt, pg, ref[-1][2][perm])
    # the next window starts from the committed page and follows the rule from there
    S1 = _dequant64(fmt, pg, perm)
    ref2 = _evolve64(S1, steps[3:])
    rec2 = _run_window(fmt, pg, perm, steps[3:], seed=9, step0=3)
    for t in range(3):
        assert _rel_l2(rec2[t][0], ref2[t][0]) <= 1e-5
    _check_commit(fmt, pg, ref2[-1][2][perm])


FORMATS_D4 = [
    ([(1, "int", 8), (2, "int", 6), (1, "int", 4)], True),
    ([(2, "fp16", 0), (2, "int", 8)], False),
    ([(4, "int", 3)], True),
]


@pytest.mark.parametrize("groups,col", FORMATS_D4)
@pytest.mark.parametrize("gate_vector", [False, True])
def test_brute_force_d4(groups, col, gate_vector):
    U = 2.0**-24
    for seed in range(6):
        rng = np.random.default_rng(100 + seed)
        fmt = O.make_format(groups, d_k=4, d_v=4, col_scales=col, gate_vector=gate_vector)
        S = (rng.normal(size=(4, 4)) * np.exp(rng.normal(size=(4, 1)))).astype(np.float32)
        perm = rng.permutation(4).astype(np.int32)
        page = O.quantize_page(fmt, S, perm)
        steps = []
        for _ in range(3):
            q, k = rng.normal(size=4).astype(np.float32), rng.normal(size=4).astype(np.float32)
            q /= np.linalg.norm(q)
            k /= np.linalg.norm(k)
            v = rng.normal(size=4).astype(np.float32)
            alpha = (1 / (1 + np.exp(rng.normal(-2, 1, size=4 if gate_vector else 1)))).astype(np.float32)
            steps.append((q, k, v, alpha, float(np.float32(1 / (1 + np.exp(-rng.normal()))))))
        S0 = _dequant64(fmt, page, perm)
        ref = _evolve64(S0, steps)
        rec = _run_window(fmt, page.copy(), perm, steps)
        scale = max(np.abs(S0).max(), max(np.abs(r[2]).max() for r in ref))
        for t in range(3):
            assert np.abs(rec[t][0] - ref[t][0]).max() <= 256 * U * scale, (seed, t)


@pytest.mark.parametrize("name", list(W.FORMATS))
def test_window_of_one_is_the_plain_step(name):
    w, fmt, perm, page = _workload(name)
    (q, k, v, alpha, beta), = _inputs(w, 11, 1)
    pa, pb = page.copy(), page.copy()
    o_step, _, mg = O.step_f32(fmt, pa, perm, q, k, v, alpha, beta, seed=5, step=2, b=1, h=3, want_margin=True)
    P = np.ones(fmt.d_k, np.float32)
    K = np.zeros((1, fmt.d_k), np.float32)
    D = np.zeros((1, fmt.d_v), np.float32)
    o_win, _ = O.window_step_f32(fmt, pb, perm, P, K, D, 0, True, q, k, v, alpha, beta, seed=5, step=2, b=1, h=3)
    assert _rel_l2(o_win, o_step) <= 2e-6
    np.testing.assert_allclose(pb.r, pa.r, rtol=2e-6)
    far = mg > 1e-3          # away from a rounding midpoint both sides round alike
    assert far.mean() > 0.99
    np.testing.assert_array_equal(pb.code[far], pa.code[far])
    assert np.abs(pb.code - pa.code).max() <= 1


@pytest.mark.parametrize("name", list(W.FORMATS))
def test_identity_window_leaves_the_page(name):
    w, fmt, perm, page = _workload(name)
    steps = [(q, k, v, np.ones_like(a), 0.0) for q, k, v, a, _ in _inputs(w, 3, 5)]
    pg = page.copy()
    rec = _run_window(fmt, pg, perm, steps, seed=1)
    np.testing.assert_array_equal(pg.code, page.code)
    np.testing.assert_array_equal(pg.r, page.r)
    assert not rec[-1][3].any()                      # no deltas
    S0 = _dequant64(fmt, page, perm)
    for t, (q, *_rest) in enumerate(steps):
        assert _rel_l2(rec[t][0], S0.T @ q.astype(np.float64)) <= 1e-6


def test_zero_gate_forgets_the_window_so_far():
    """alpha = 0 at step 2: the state after it is beta k (v)^T alone, as if
    the page and the first two entries had never been."""
    w, fmt, perm, page = _workload("stepquant6")
    steps = _inputs(w, 90, 4)
    q, k, v, alpha, beta = steps[2]
    steps[2] = (q, k, v, np.zeros_like(alpha), beta)
    rec = _run_window(fmt, page.copy(), perm, steps)
    S2 = float(beta) * np.outer(k.astype(np.float64), v.astype(np.float64))
    assert _rel_l2(rec[2][0], S2.T @ q.astype(np.float64)) <= 1e-6
    assert not rec[2][1].any() and not rec[2][2][:2].any()
    S_ref = _evolve64(S2, steps[3:])
    assert _rel_l2(rec[3][0], S_ref[0][0]) <= 1e-5


def test_first_step_of_a_window_reads_no_decay():
    """At t = 0 the cumulative decay starts from one whatever the buffer holds."""
    w, fmt, perm, page = _workload("stepquant4_kda")
    (q, k, v, alpha, beta), = _inputs(w, 5, 1)
    outs = []
    for P0 in (np.ones(fmt.d_k, np.float32), np.full(fmt.d_k, 7.5, np.float32)):
        P = P0.copy()
        K = np.zeros((2, fmt.d_k), np.float32)
        D = np.zeros((2, fmt.d_v), np.float32)
        o, _ = O.window_step_f32(fmt, page.copy(), perm, P, K, D, 0, False, q, k, v, alpha, beta)
        outs.append((o, P))
    np.testing.assert_array_equal(outs[0][0], outs[1][0])
    np.testing.assert_array_equal(outs[1][1], np.atleast_1d(alpha).astype(np.float32) * np.ones(fmt.d_k, np.float32))
