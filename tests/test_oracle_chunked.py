"""Pins of the chunkwise prefill's algebra (orc_prefill_chunked_f64).

A tensor-core prefill runs a prompt chunk by chunk: per chunk the keys'
interactions are resolved by the triangular solve (I + A)^-1 and everything
else is matrix products (repeated prefill: DASC card page; the delta rule of
the dev.to post, "The state is a running sum, not a buffer", with gate and
write strength).  In exact arithmetic this reproduces the token recurrence,
so the oracle's fp64 chunk algebra is pinned against the recurrence written
out here token by token in numpy (fp64), for chunk sizes that divide the
prompt, leave a ragged last chunk, are one token, or are the whole prompt;
GDN and KDA gates; 4 x 4 brute force and full 128 x 128 pages.  Also: the
chunked o and state agree with the oracle's own fp32 prefill to fp32
rounding, and a single token is the fp64 decode step.
"""
import numpy as np
import pytest

import oracle as O
from linear_attention_recurrent_delta_b200 import workloads as W

from test_oracle_prefill import _dequant64, _evolve64, _prompt, _rel_l2, _workload


@pytest.mark.parametrize("name", ["stepquant6", "stepquant4_kda", "damp"])
@pytest.mark.parametrize("L,C", [(64, 64), (100, 32), (37, 1), (37, 37), (130, 64)])
def test_chunk_algebra_is_the_recurrence(name, L, C):
    w, fmt, perm, page = _workload(name)
    q, k, v, alpha, beta = _prompt(w, 11, L)
    o64, S64 = _evolve64(_dequant64(fmt, page, perm), q, k, v, alpha, beta)
    oc, Sc = O.prefill_chunked_f64(fmt, page, perm, q, k, v, alpha, beta, C)
    assert _rel_l2(oc, o64) <= 1e-12, _rel_l2(oc, o64)
    assert _rel_l2(Sc, S64) <= 1e-12, _rel_l2(Sc, S64)


@pytest.mark.parametrize("gate_vector", [False, True])
@pytest.mark.parametrize("C", [1, 2, 3, 5])
def test_brute_force_d4(gate_vector, C):
    for seed in range(6):
        rng = np.random.default_rng(300 + seed)
        fmt = O.make_format([(2, "int", 8), (2, "int", 4)], d_k=4, d_v=4, col_scales=True,
                            gate_vector=gate_vector)
        S0 = rng.standard_normal((4, 4)).astype(np.float32)
        perm = rng.permutation(4).astype(np.int32)
        page = O.quantize_page(fmt, S0, perm)
        L = 5
        q = rng.standard_normal((L, 4)).astype(np.float32)
        k = rng.standard_normal((L, 4)).astype(np.float32)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
        v = rng.standard_normal((L, 4)).astype(np.float32)
        alpha = rng.uniform(0.3, 1.0, (L, 4 if gate_vector else 1)).astype(np.float32)
        beta = rng.uniform(0.1, 1.0, L).astype(np.float32)
        o64, S64 = _evolve64(_dequant64(fmt, page, perm), q, k, v, alpha, beta)
        oc, Sc = O.prefill_chunked_f64(fmt, page, perm, q, k, v, alpha, beta, C)
        np.testing.assert_allclose(oc, o64, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(Sc, S64, rtol=1e-12, atol=1e-12)


def test_one_token_is_the_f64_step():
    w, fmt, perm, page = _workload("stepquant6")
    q, k, v, alpha, beta = _prompt(w, 5, 1)
    o1, S1 = O.step_f64(fmt, page, perm, q[0], k[0], v[0], alpha[0], float(beta[0]))
    oc, Sc = O.prefill_chunked_f64(fmt, page, perm, q, k, v, alpha, beta, 64)
    np.testing.assert_allclose(oc[0], o1, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(Sc, S1, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("name", ["int8row", "stepquant4_kda"])
def test_chunked_f64_and_the_f32_prefill_agree(name):
    w, fmt, perm, page = _workload(name)
    q, k, v, alpha, beta = _prompt(w, 40, 96)
    oc, Sc = O.prefill_chunked_f64(fmt, page, perm, q, k, v, alpha, beta, 64)
    pg = page.copy()
    o32, tp, _ = O.prefill_f32(fmt, pg, perm, q, k, v, alpha, beta, want_tp=True, plain=True)
    assert _rel_l2(o32, oc) <= 1e-5
    c = page.c.astype(np.float64) if fmt.col_scales else np.ones(128)
    S32 = np.zeros_like(Sc)
    S32[perm] = tp.astype(np.float64) * c
    assert _rel_l2(S32, Sc) <= 1e-5


@pytest.mark.parametrize("name", ["stepquant6", "stepquant4_kda"])
def test_zero_and_vanishing_gates(name):
    """Gates of zero, and runs of small gates whose cumulative product leaves
    the double range within a chunk (0.002^128 ~ 1e-345), still give the
    recurrence: the decay between two tokens is a product of gates, never a
    quotient of cumulative decays."""
    w, fmt, perm, page = _workload(name)
    L, C = 200, 128
    q, k, v, alpha, beta = _prompt(w, 17, L)
    alpha = alpha.copy()
    alpha[5] = 0.0                      # one token forgets everything
    alpha[20:150] = 0.002               # the cumulative decay underflows double
    if alpha.shape[1] > 1:
        alpha[60, ::3] = 0.0            # KDA: some channels only
    o64, S64 = _evolve64(_dequant64(fmt, page, perm), q, k, v, alpha, beta)
    oc, Sc = O.prefill_chunked_f64(fmt, page, perm, q, k, v, alpha, beta, C)
    assert np.all(np.isfinite(oc)) and np.all(np.isfinite(Sc))
    assert _rel_l2(oc, o64) <= 1e-12, _rel_l2(oc, o64)
    assert _rel_l2(Sc, S64) <= 1e-12, _rel_l2(Sc, S64)
