"""Pins of the oracle's decode step.

* fp64 plain mode against the explicit matrix form (numpy matmul), including
  the pages' own d_v x d_k form S <- S(I - k k^T) + v k^T (dev.to post, "The
  state is a running sum, not a buffer"), at d = 4 and d = 128, GDN and KDA;
* canonical fp32 mode against fp64 mode (rel-L2 <= 1e-5 on o and on the
  pre-rounding state, every format, workload distributions);
* invariants of the method: alpha = 1, beta = 0 leaves the state unchanged;
  unquantized fp32 state, alpha = beta = 1, |k| = 1, q = k reads out v;
* closed forms: beta = 0 is pure decay, alpha = 0 leaves beta k v^T;
* special cases: KDA with equal alphas == GDN, bit for bit; column scales
  all one == no column scales, bit for bit;
* stochastic rounding: only floor/ceil outcomes, unbiased, deterministic.
"""
import numpy as np
import pytest

import oracle as O
from linear_attention_recurrent_delta_b200 import workloads as W

U = 2.0**-24


def _rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def _dequant64(fmt, page, perm):
    """q_ij * r_i * c_j in double, natural key order."""
    d_k, d_v = fmt.d_k, fmt.d_v
    S = np.zeros((d_k, d_v))
    for s in range(d_k):
        kind = O.row_kind(fmt, s)
        if kind == 0:
            x = page.code[s].astype(np.float64) * float(page.r[s])
        elif kind == 1:
            x = O.f16_to_f32(page.code[s].astype(np.uint16)).astype(np.float64)
        else:
            x = page.code[s].astype(np.uint32).view(np.float32).astype(np.float64)
        S[perm[s]] = x * (page.c.astype(np.float64) if fmt.col_scales else 1.0)
    return S


def _random_case(fmt, rng, gate_vector):
    d_k, d_v = fmt.d_k, fmt.d_v
    S = (rng.normal(size=(d_k, d_v)) * np.exp(rng.normal(size=(d_k, 1)))
         * np.exp(rng.normal(size=(1, d_v)))).astype(np.float32)
    perm = rng.permutation(d_k).astype(np.int32)
    page = O.quantize_page(fmt, S, perm)
    q = rng.normal(size=d_k).astype(np.float32)
    k = rng.normal(size=d_k).astype(np.float32)
    q /= np.linalg.norm(q)
    k /= np.linalg.norm(k)
    v = rng.normal(size=d_v).astype(np.float32)
    alpha = (1 / (1 + np.exp(rng.normal(-4, 1.5, size=d_k if gate_vector else 1)))).astype(np.float32)
    beta = np.float32(1 / (1 + np.exp(-rng.normal())))
    return page, perm, q, k, v, alpha, beta


FORMATS_D4 = [
    ([(1, "int", 8), (2, "int", 6), (1, "int", 4)], True),
    ([(2, "fp16", 0), (2, "int", 8)], False),
    ([(4, "int", 3)], True),
]


@pytest.mark.parametrize("groups,col", FORMATS_D4)
@pytest.mark.parametrize("gate_vector", [False, True])
@pytest.mark.parametrize("seed", range(4))
def test_f64_step_is_the_matrix_form_d4(groups, col, gate_vector, seed):
    fmt = O.make_format(groups, d_k=4, d_v=4, col_scales=col, gate_vector=gate_vector)
    rng = np.random.default_rng(seed)
    page, perm, q, k, v, alpha, beta = _random_case(fmt, rng, gate_vector)
    S = _dequant64(fmt, page, perm)
    A = np.diag(alpha.astype(np.float64)) if gate_vector else float(alpha[0]) * np.eye(4)
    k64, q64, v64 = k.astype(np.float64), q.astype(np.float64), v.astype(np.float64)
    Sp = (np.eye(4) - float(beta) * np.outer(k64, k64)) @ A @ S + float(beta) * np.outer(k64, v64)
    o64, sp64 = O.step_f64(fmt, page, perm, q, k, v, alpha, beta)
    np.testing.assert_allclose(sp64, Sp, rtol=1e-12, atol=1e-12 * np.abs(Sp).max())
    np.testing.assert_allclose(o64, Sp.T @ q64, rtol=1e-12, atol=1e-12 * np.abs(Sp).max())


def test_f64_step_is_the_pages_transposed_formula():
    """dev.to post: S <- S(I - k k^T) + v k^T with the state d_v x d_k
    (alpha = beta = 1); the library's state is its transpose."""
    fmt = O.make_format([(128, "int", 8)], col_scales=True)
    rng = np.random.default_rng(11)
    page, perm, q, k, v, _, _ = _random_case(fmt, rng, False)
    St = _dequant64(fmt, page, perm).T                       # d_v x d_k
    k64 = k.astype(np.float64)
    St_new = St @ (np.eye(128) - np.outer(k64, k64)) + np.outer(v.astype(np.float64), k64)
    _, sp64 = O.step_f64(fmt, page, perm, q, k, v, np.float32(1), np.float32(1))
    np.testing.assert_allclose(sp64.T, St_new, rtol=1e-11, atol=1e-11 * np.abs(St_new).max())


def _workload_case(name, rng):
    w = [x for x in W.WORKLOADS if x.fmt == name][0]
    fmt = O.format_from_spec(W.FORMATS[name])
    S = W.initial_state(w, batch=1)[:, :1].numpy()
    perm = O.rank_rows(fmt, S)[0]
    page = O.quantize_page(fmt, S[0, 0], perm)
    x = W.step_inputs(w, int(rng.integers(1000)), batch=1)
    return (w, fmt, page, perm, x["q"][0, 0].numpy(), x["k"][0, 0].numpy(), x["v"][0, 0].numpy(),
            x["alpha"][0, 0].numpy(), float(x["beta"][0, 0]))


@pytest.mark.parametrize("plain", [False, True])
@pytest.mark.parametrize("name", list(W.FORMATS))
def test_canonical_f32_matches_f64_definition(name, plain):
    """Both fp32 evaluations (the kernel's canonical order and the plain
    natural-order chains) follow the fp64 definition to rel-L2 1e-5."""
    rng = np.random.default_rng(21)
    w, fmt, page, perm, q, k, v, alpha, beta = _workload_case(name, rng)
    for step in range(8):
        o64, sp64 = O.step_f64(fmt, page, perm, q, k, v, alpha, beta)
        o32, tp, _ = O.step_f32(fmt, page, perm, q, k, v, alpha, beta, seed=3, step=step,
                                want_tp=True, plain=plain)
        sp32 = np.zeros_like(sp64)
        sp32[perm] = tp.astype(np.float64) * (page.c.astype(np.float64) if fmt.col_scales else 1.0)
        assert _rel_l2(o32, o64) <= 1e-5
        assert _rel_l2(sp32, sp64) <= 1e-5
        # fresh inputs for the next step, state carried
        x = W.step_inputs(w, 500 + step, batch=1)
        q, k, v = (x[n][0, 0].numpy() for n in ("q", "k", "v"))
        alpha, beta = x["alpha"][0, 0].numpy(), float(x["beta"][0, 0])


@pytest.mark.parametrize("plain", [False, True])
@pytest.mark.parametrize("gate_vector", [False, True])
def test_canonical_f32_matches_f64_d4(gate_vector, plain):
    for seed in range(20):
        fmt = O.make_format(FORMATS_D4[0][0], d_k=4, d_v=4, col_scales=True, gate_vector=gate_vector)
        page, perm, q, k, v, alpha, beta = _random_case(fmt, np.random.default_rng(seed), gate_vector)
        o64, sp64 = O.step_f64(fmt, page, perm, q, k, v, alpha, beta)
        o32, tp, _ = O.step_f32(fmt, page, perm, q, k, v, alpha, beta, want_tp=True, plain=plain)
        sp32 = np.zeros_like(sp64)
        sp32[perm] = tp.astype(np.float64) * page.c
        scale = np.abs(sp64).max()
        assert np.abs(sp32 - sp64).max() <= 64 * U * scale
        assert np.abs(o32 - o64).max() <= 64 * U * scale * 4


@pytest.mark.parametrize("name", ["stepquant6", "int8row", "stepquant4_kda"])
def test_identity_step_leaves_the_state_unchanged(name):
    """Invariant: alpha = 1, beta = 0 leaves the dequantized state
    unchanged.  The row scale is re-derived from the row's absmax, so codes
    stay bit-identical and r moves by at most one ulp."""
    rng = np.random.default_rng(4)
    w, fmt, page, perm, q, k, v, _, _ = _workload_case(name, rng)
    before = page.copy()
    ones = np.ones(128 if fmt.gate_vector else 1, np.float32)
    for step in range(5):
        O.step_f32(fmt, page, perm, q, k, v, ones, 0.0, step=step)
        np.testing.assert_array_equal(page.code, before.code)
        ulp = np.spacing(before.r)
        assert np.all(np.abs(page.r - before.r) <= ulp)
        np.testing.assert_array_equal(page.c, before.c)


def test_identity_step_damp_format():
    """Same invariant on the DAMP-style format: FP16 rows are bit-identical;
    INT8 rows under stochastic rounding keep their codes except where the
    offset delta falls within the scale's rounding slack of +-1/2."""
    rng = np.random.default_rng(6)
    w, fmt, page, perm, q, k, v, _, _ = _workload_case("damp", rng)
    before = page.copy()
    o, _, margin = O.step_f32(fmt, page, perm, q, k, v, np.float32(1), 0.0, seed=77, step=1,
                              want_margin=True)
    np.testing.assert_array_equal(page.code[:16], before.code[:16])
    diff = page.code[16:] != before.code[16:]
    assert np.all(np.abs(page.code[16:] - before.code[16:])[diff] == 1)
    assert np.all(margin[16:][diff] < 1e-4)
    assert diff.sum() <= 8


def test_unquantized_state_retrieves_v():
    """Invariant: unquantized fp32 state, alpha = beta = 1,
    |k| = 1: reading out at q = k returns v (exact in the fp64 definition;
    within the fp32 rounding bound in the canonical evaluation)."""
    fmt = O.make_format([(128, "fp32", 0)])
    rng = np.random.default_rng(8)
    for trial in range(10):
        S = (rng.normal(size=(128, 128)) * np.exp(rng.normal(size=(128, 1)))).astype(np.float32)
        perm = rng.permutation(128).astype(np.int32)
        page = O.quantize_page(fmt, S, perm)
        np.testing.assert_array_equal(O.dequantize_page(fmt, page, perm), S)
        k = rng.normal(size=128)
        k = (k / np.linalg.norm(k)).astype(np.float32)
        v = rng.normal(size=128).astype(np.float32)
        kk = float(np.dot(k.astype(np.float64), k.astype(np.float64)))
        o64, sp64 = O.step_f64(fmt, page, perm, k, k, v, np.float32(1), np.float32(1))
        pred = S.astype(np.float64).T @ k.astype(np.float64)
        # exact algebra: S'^T k = S^T k + (v - S^T k)(k^T k)
        np.testing.assert_allclose(o64, pred + (v - pred) * kk, rtol=0, atol=1e-12 * np.abs(S).max())
        assert np.abs(o64 - v).max() <= abs(kk - 1) * np.abs(v - pred).max() + 1e-11 * np.abs(S).max()
        o32, tp, _ = O.step_f32(fmt, page, perm, k, k, v, np.float32(1), np.float32(1), want_tp=True)
        sp = np.zeros((128, 128))
        sp[perm] = tp
        mag = np.abs(k.astype(np.float64)) @ (np.abs(S) + np.abs(sp))
        bound = 80 * U * mag + abs(kk - 1) * np.abs(v - pred) + U * np.abs(v)
        assert np.all(np.abs(o32 - v) <= bound)


@pytest.mark.parametrize("name", ["stepquant6", "stepquant4_kda"])
def test_beta_zero_is_pure_decay_and_alpha_zero_writes_kv(name):
    rng = np.random.default_rng(9)
    w, fmt, page, perm, q, k, v, alpha, beta = _workload_case(name, rng)
    S = _dequant64(fmt, page, perm)
    alpha = np.atleast_1d(alpha)
    A = alpha.astype(np.float64)[:, None] if fmt.gate_vector else float(alpha[0])
    _, sp = O.step_f64(fmt, page, perm, q, k, v, alpha, 0.0)
    np.testing.assert_allclose(sp, A * S, rtol=1e-15, atol=0)
    zero = np.zeros_like(alpha)
    o, sp = O.step_f64(fmt, page, perm, q, k, v, zero, beta)
    kv = beta * np.outer(k.astype(np.float64), v.astype(np.float64))
    np.testing.assert_allclose(sp, kv, rtol=1e-15, atol=0)
    expect = beta * float(np.dot(k.astype(np.float64), q.astype(np.float64))) * v.astype(np.float64)
    np.testing.assert_allclose(o, expect, rtol=1e-12)


def test_kda_with_equal_alphas_is_gdn_bit_for_bit():
    rng = np.random.default_rng(12)
    spec = dict(W.FORMATS["stepquant4_kda"])
    fmt_kda = O.format_from_spec(spec)
    fmt_gdn = O.format_from_spec(dict(spec, gate_vector=False))
    w, _, page, perm, q, k, v, _, beta = _workload_case("stepquant4_kda", rng)
    a = np.float32(0.97)
    p1, p2 = page.copy(), page.copy()
    o1, _, _ = O.step_f32(fmt_kda, p1, perm, q, k, v, np.full(128, a, np.float32), beta)
    o2, _, _ = O.step_f32(fmt_gdn, p2, perm, q, k, v, np.float32(a), beta)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(p1.code, p2.code)
    np.testing.assert_array_equal(p1.r, p2.r)


def test_unit_column_scales_equal_no_column_scales_bit_for_bit():
    rng = np.random.default_rng(13)
    spec = dict(W.FORMATS["stepquant6"])
    fmt_c = O.format_from_spec(spec)
    fmt_n = O.format_from_spec(dict(spec, col_scales=False))
    w, _, page, perm, q, k, v, alpha, beta = _workload_case("stepquant6", rng)
    page.c[:] = 1
    p1, p2 = page.copy(), page.copy()
    o1, _, _ = O.step_f32(fmt_c, p1, perm, q, k, v, alpha, beta)
    o2, _, _ = O.step_f32(fmt_n, p2, perm, q, k, v, alpha, beta)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(p1.code, p2.code)
    np.testing.assert_array_equal(p1.r, p2.r)


def test_stochastic_rounding_floor_ceil_unbiased_deterministic():
    rng = np.random.default_rng(14)
    w, fmt, page, perm, q, k, v, alpha, beta = _workload_case("damp", rng)
    n_seeds = 1024
    acc = np.zeros((112, 128))
    first = None
    for seed in range(n_seeds):
        p = page.copy()
        _, tp, _ = O.step_f32(fmt, p, perm, q, k, v, alpha, beta, seed=seed, step=3, want_tp=True)
        x = tp[16:].astype(np.float64) / p.r[16:].astype(np.float64)[:, None]
        z = p.code[16:]
        # outcomes: floor or ceil of the scaled value only
        assert np.all((z == np.floor(x)) | (z == np.ceil(x)) | (np.abs(z - x) < 1e-3))
        acc += z
        if first is None:
            first = z.copy()
            x_ref = x
    mean = acc / n_seeds
    frac = x_ref - np.floor(x_ref)
    sigma = np.sqrt(np.maximum(frac * (1 - frac), 1e-4) / n_seeds)
    # unbiased: the mean code tracks the scaled value
    assert np.mean(np.abs(mean - x_ref) <= 4.5 * sigma + 1e-3) > 0.999
    p = page.copy()
    O.step_f32(fmt, p, perm, q, k, v, alpha, beta, seed=0, step=3)
    np.testing.assert_array_equal(p.code[16:], first)
