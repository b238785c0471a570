"""Pins of the oracle's prefill (orc_prefill_f32): a prompt of L tokens run
through one page in fp32, requantized once at the end.

* L = 1 is the decode step, bit for bit (o, codes, r), every format;
* o at every token and the final state before requantization against the
  gated delta rule in fp64 (numpy) from the dequantized page, rel-L2 <= 1e-5,
  every format, L = 32; the requantized page within one quantization step of
  the fp64 state (half a step for round to nearest);
* alpha = 1, beta = 0 over a prompt leaves the page (codes identical, row
  scales within one ulp);
* from a zero state: one token gives o = beta (q . k) v; writing values under
  orthonormal (basis) keys with alpha = beta = 1 and reading them back
  returns them to rounding.
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
    S = np.zeros((fmt.d_k, fmt.d_v))
    for s in range(fmt.d_k):
        kind = O.row_kind(fmt, s)
        if kind == 0:
            x = page.code[s].astype(np.float64) * float(page.r[s])
        else:
            x = O.f16_to_f32(page.code[s].astype(np.uint16)).astype(np.float64)
        S[perm[s]] = x * (page.c.astype(np.float64) if fmt.col_scales else 1.0)
    return S


def _workload(name):
    w = [x for x in W.WORKLOADS if x.fmt == name][0]
    fmt = O.format_from_spec(W.FORMATS[name])
    S = W.initial_state(w, batch=1)[:, :1].numpy()
    perm = O.rank_rows(fmt, S)[0]
    page = O.quantize_page(fmt, S[0, 0], perm)
    return w, fmt, perm, page


def _prompt(w, first, L):
    xs = [W.step_inputs(w, first + i, batch=1) for i in range(L)]
    q, k, v = (np.stack([x[n][0, 0].numpy() for x in xs]) for n in ("q", "k", "v"))
    alpha = np.stack([np.atleast_1d(x["alpha"][0, 0].numpy()) for x in xs])
    beta = np.array([float(x["beta"][0, 0]) for x in xs], np.float32)
    return q, k, v, alpha, beta


def _evolve64(S0, q, k, v, alpha, beta):
    S = S0.copy()
    outs = []
    for l in range(len(q)):
        a = alpha[l].astype(np.float64)
        S = (a[:, None] if a.size > 1 else float(a[0])) * S
        k64 = k[l].astype(np.float64)
        S = S + float(beta[l]) * np.outer(k64, v[l].astype(np.float64) - S.T @ k64)
        outs.append(S.T @ q[l].astype(np.float64))
    return np.array(outs), S


@pytest.mark.parametrize("name", list(W.FORMATS))
def test_one_token_is_the_decode_step(name):
    w, fmt, perm, page = _workload(name)
    q, k, v, alpha, beta = _prompt(w, 7, 1)
    pa, pb = page.copy(), page.copy()
    o1, _, _ = O.step_f32(fmt, pa, perm, q[0], k[0], v[0], alpha[0], float(beta[0]), seed=4, step=9, b=2, h=1)
    o2, _, _ = O.prefill_f32(fmt, pb, perm, q, k, v, alpha, beta, seed=4, step=9, b=2, h=1)
    assert np.array_equal(o1, o2[0])
    assert np.array_equal(pa.code, pb.code)
    assert np.array_equal(pa.r, pb.r)


@pytest.mark.parametrize("plain", [False, True])
@pytest.mark.parametrize("name", list(W.FORMATS))
def test_prompt_follows_the_f64_rule(name, plain):
    w, fmt, perm, page = _workload(name)
    q, k, v, alpha, beta = _prompt(w, 30, 32)
    S0 = _dequant64(fmt, page, perm)
    o64, S64 = _evolve64(S0, q, k, v, alpha, beta)
    pg = page.copy()
    o, tp, _ = O.prefill_f32(fmt, pg, perm, q, k, v, alpha, beta, want_tp=True, plain=plain)
    for l in range(len(q)):
        assert _rel_l2(o[l], o64[l]) <= 1e-5, (l, _rel_l2(o[l], o64[l]))
    c = page.c.astype(np.float64) if fmt.col_scales else np.ones(fmt.d_v)
    S32 = np.zeros_like(S64)
    S32[perm] = tp.astype(np.float64) * c
    assert _rel_l2(S32, S64) <= 1e-5
    # the one requantization: each element within one step of its new row scale
    Sq = _dequant64(fmt, pg, np.arange(fmt.d_k))
    ref = S64[perm]
    for s in range(fmt.d_k):
        if O.row_kind(fmt, s) == 0:
            unit = float(pg.r[s]) * c
            frac = 1.0 if fmt.stochastic else 0.5
            assert np.all(np.abs(Sq[s] - ref[s]) <= (frac + 1e-3) * unit + 1e-6 * np.abs(ref[s])), s


@pytest.mark.parametrize("name", ["stepquant6", "damp"])
def test_identity_prompt_leaves_the_page(name):
    w, fmt, perm, page = _workload(name)
    q, k, v, alpha, beta = _prompt(w, 3, 6)
    pg = page.copy()
    O.prefill_f32(fmt, pg, perm, q, k, v, np.ones_like(alpha), np.zeros_like(beta))
    assert np.array_equal(pg.code, page.code)
    assert np.all(np.abs(pg.r.view(np.int32) - page.r.view(np.int32)) <= 1)


def _zero_page(fmt):
    perm = np.arange(fmt.d_k, dtype=np.int32)
    return perm, O.quantize_page(fmt, np.zeros((fmt.d_k, fmt.d_v), np.float32), perm)


def test_one_token_from_a_zero_state():
    fmt = O.format_from_spec(W.FORMATS["int8row"])
    perm, page = _zero_page(fmt)
    rng = np.random.default_rng(5)
    q, k, v = (rng.normal(size=(1, 128)).astype(np.float32) for _ in range(3))
    o, _, _ = O.prefill_f32(fmt, page, perm, q, k, v, np.array([0.9], np.float32), np.array([0.5], np.float32))
    ref = 0.5 * float(q[0].astype(np.float64) @ k[0].astype(np.float64)) * v[0].astype(np.float64)
    assert _rel_l2(o[0], ref) <= 1e-6


def test_basis_keys_store_and_return_values():
    fmt = O.format_from_spec(W.FORMATS["stepquant6"])    # mixed widths; a zero state's column scales are 1
    perm, page = _zero_page(fmt)
    rng = np.random.default_rng(9)
    idx = rng.permutation(128)[:24]
    L = len(idx) + 1
    k = np.zeros((L, 128), np.float32)
    k[np.arange(len(idx)), idx] = 1.0
    v = rng.normal(size=(L, 128)).astype(np.float32)
    q = np.zeros((L, 128), np.float32)
    q[:-1] = k[:-1]
    q[-1, idx[3]] = 1.0                                 # read back the value written under key 3
    alpha = np.ones((L, 1), np.float32)
    beta = np.ones(L, np.float32)
    beta[-1] = 0.0
    o, _, _ = O.prefill_f32(fmt, page, perm, q, k, v, alpha, beta)
    for l in range(len(idx)):
        np.testing.assert_allclose(o[l], v[l], rtol=4e-7, atol=1e-30)
    np.testing.assert_allclose(o[-1], v[3], rtol=4e-7, atol=1e-30)


@pytest.mark.parametrize("name", ["stepquant6", "stepquant4_kda"])
def test_prefill_and_a_window_of_the_same_steps_agree(name):
    """A window of L steps and a prefill of the same L tokens run the same
    exact rule in two fp32 orders: o of every token, and the state before the
    one requantization (the window's rebuilt from its buffer), agree to
    rounding."""
    w, fmt, perm, page = _workload(name)
    L = 8
    q, k, v, alpha, beta = _prompt(w, 60, L)
    o_p, tp, _ = O.prefill_f32(fmt, page.copy(), perm, q, k, v, alpha, beta, want_tp=True)
    P = np.ones(128, np.float32)
    K = np.zeros((L, 128), np.float32)
    D = np.zeros((L, 128), np.float32)
    pw = page.copy()
    for t in range(L):
        o_w, _ = O.window_step_f32(fmt, pw, perm, P, K, D, t, False, q[t], k[t], v[t], alpha[t], float(beta[t]))
        assert _rel_l2(o_w, o_p[t]) <= 1e-5, t
    # the window's state after step L - 1, rebuilt in fp64 from its buffer: P' S0 + sum K D^T
    S0 = _dequant64(fmt, page, perm)
    c = page.c.astype(np.float64) if fmt.col_scales else np.ones(128)
    Sw = P.astype(np.float64)[:, None] * S0 + (K.astype(np.float64).T @ D.astype(np.float64)) * c[None, :]
    Sp = np.zeros((128, 128))
    Sp[perm] = tp.astype(np.float64) * c
    assert _rel_l2(Sw, Sp) <= 1e-5


FORMATS_D4 = [
    ([(1, "int", 8), (2, "int", 6), (1, "int", 4)], True),
    ([(2, "fp16", 0), (2, "int", 8)], False),
    ([(4, "int", 3)], True),
]


@pytest.mark.parametrize("groups,col", FORMATS_D4)
@pytest.mark.parametrize("gate_vector", [False, True])
def test_brute_force_d4(groups, col, gate_vector):
    """4 x 4 states, five tokens: every token's o against the fp64 rule
    within a few ulps of the state's scale."""
    U = 2.0**-24
    for seed in range(6):
        rng = np.random.default_rng(300 + seed)
        fmt = O.make_format(groups, d_k=4, d_v=4, col_scales=col, gate_vector=gate_vector)
        S = (rng.normal(size=(4, 4)) * np.exp(rng.normal(size=(4, 1)))).astype(np.float32)
        perm = rng.permutation(4).astype(np.int32)
        page = O.quantize_page(fmt, S, perm)
        L = 5
        q = rng.normal(size=(L, 4)).astype(np.float32)
        k = rng.normal(size=(L, 4)).astype(np.float32)
        q /= np.linalg.norm(q, axis=1, keepdims=True)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
        v = rng.normal(size=(L, 4)).astype(np.float32)
        alpha = (1 / (1 + np.exp(rng.normal(-2, 1, size=(L, 4 if gate_vector else 1))))).astype(np.float32)
        beta = (1 / (1 + np.exp(-rng.normal(size=L)))).astype(np.float32)
        S0 = _dequant64(fmt, page, perm)
        o64, S64 = _evolve64(S0, q, k, v, alpha, beta)
        o, tp, _ = O.prefill_f32(fmt, page.copy(), perm, q, k, v, alpha, beta, want_tp=True)
        scale = max(np.abs(S0).max(), np.abs(S64).max(), 1.0)
        assert np.abs(o - o64).max() <= 256 * U * scale, seed
