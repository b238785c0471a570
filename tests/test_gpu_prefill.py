"""GPU parity of the prefill (stq_prefill) with the oracle's orc_prefill_f32.

Both sides start from the same packed pages and take the same prompt.  Bar:
o of every token bit-identical, the optional fp32 state (S = T c, natural
key order) bit-identical, the requantized pages bit-identical except codes
whose pre-rounding value the oracle reports within 1e-5 (relative) of a
rounding boundary.  L = 1 is also checked against the decode step.
"""
import numpy as np
import pytest
import torch

import oracle as O
from linear_attention_recurrent_delta_b200 import binding as B
from linear_attention_recurrent_delta_b200 import workloads as W

from parity_util import BAND, download, make_state, oracle_quantize, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from linear_attention_recurrent_delta_b200 import build
    build.build()
    B.lib()
    assert torch.cuda.is_available()


def _setup(name, batch, heads, zero=False):
    base = [w for w in W.WORKLOADS if w.fmt == name and w.index > 0][0]
    w = W.Workload(base.index, base.name, name, batch, heads, 2, base.gate_mu, base.gate_sigma, base.seed)
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    if zero:   # a zero state quantized with the same map: codes 0, r = 0, c = 1
        pages = np.stack([O.pack_page(fmt, O.quantize_page(fmt, np.zeros((128, 128), np.float32), perm[i % heads]))
                          for i in range(batch * heads)])
    qs = make_state(w)
    upload(qs, perm, pages)
    return w, fmt, perm, pages, qs


def _prompt(w, L, first=0):
    xs = [W.step_inputs(w, first + l) for l in range(L)]
    return {k: torch.stack([x[k] for x in xs]).contiguous() for k in xs[0]}


def _oracle(fmt, perm, pages, heads, x, seed, step):
    n, L = len(pages), x["q"].shape[0]
    arr = {k: v.numpy().reshape(L, n, -1) for k, v in x.items()}
    o = np.zeros((L, n, 128), np.float32)
    out, tps, margins = pages.copy(), [], []
    for i in range(n):
        b, h = divmod(i, heads)
        pg = O.unpack_page(fmt, pages[i])
        o_i, tp, mg = O.prefill_f32(fmt, pg, perm[h], arr["q"][:, i], arr["k"][:, i], arr["v"][:, i],
                                    arr["alpha"][:, i], arr["beta"][:, i, 0], seed=seed, step=step, b=b, h=h,
                                    want_tp=True, want_margin=True)
        o[:, i] = o_i
        out[i] = O.pack_page(fmt, pg)
        c = pg.c if fmt.col_scales else np.ones(128, np.float32)
        S_nat = np.zeros((128, 128), np.float32)
        S_nat[perm[h]] = tp * c[None, :]
        tps.append(S_nat)
        margins.append(mg)
    return out, o, np.stack(tps), margins


def _check_pages(fmt, got, ref, margins):
    for i in range(len(ref)):
        if np.array_equal(got[i], ref[i]):
            continue
        pg, pe = O.unpack_page(fmt, got[i]), O.unpack_page(fmt, ref[i])
        assert np.array_equal(pg.r.view(np.uint32), pe.r.view(np.uint32)), "r of page %d" % i
        bad = pg.code != pe.code
        assert np.all(margins[i][bad] < BAND), "codes of page %d outside the rounding band" % i


def _run(name, batch, heads, L, zero=False, with_state=True, seed_off=0):
    w, fmt, perm, pages, qs = _setup(name, batch, heads, zero)
    x = _prompt(w, L, seed_off)
    xd = {k: v.cuda() for k, v in x.items()}
    o = torch.empty(L, batch, heads, 128, device="cuda")
    S_out = torch.empty(batch, heads, 128, 128, device="cuda") if with_state else None
    seed = W.sr_seed(w)
    B.stq_prefill(qs.state, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o, S_out, seed=seed, step=5)
    assert B.stq_device_status(qs.state) == B.STQ_OK
    ref, o_ref, S_ref, margins = _oracle(fmt, perm, pages, heads, x, seed, 5)
    n = batch * heads
    assert np.array_equal(o.cpu().numpy().reshape(L, n, 128), o_ref)
    if with_state:
        assert np.array_equal(S_out.cpu().numpy().reshape(n, 128, 128), S_ref)
    _check_pages(fmt, download(qs), ref, margins)
    return w, fmt, perm, pages, qs, x


@pytest.mark.parametrize("name", ["stepquant6", "int8row", "stepquant4_kda", "damp"])
@pytest.mark.parametrize("L", [1, 7, 33])
def test_prefill_matches_oracle(name, L):
    _run(name, 9, 5, L)


def test_many_pages_per_cta_and_no_state_output():
    # more pages than resident CTAs: both page buffers and the token ring cycle across pages
    _run("int8row", 96, 20, 6, with_state=False)


@pytest.mark.parametrize("name", ["int8row", "stepquant4_kda"])
def test_prefill_from_a_zero_state(name):
    _run(name, 6, 4, 12, zero=True)


@pytest.mark.parametrize("stochastic", [False, True])
def test_runtime_format(stochastic, monkeypatch):
    name = "prefill_runtime_%d" % stochastic
    spec = {"groups": [(32, "int", 7), (16, "fp16", 0), (48, "int", 5), (32, "int", 2)], "col_scales": True,
            "gate_vector": True, "stochastic": stochastic}
    monkeypatch.setitem(W.FORMATS, name, spec)
    kda = [w for w in W.WORKLOADS if w.fmt == "stepquant4_kda"][0]
    monkeypatch.setattr(W, "WORKLOADS", list(W.WORKLOADS) + [
        W.Workload(kda.index, name, name, 5, 4, 2, kda.gate_mu, kda.gate_sigma, kda.seed + 3)])
    _run(name, 5, 4, 9)


def test_one_token_is_the_decode_step():
    w, fmt, perm, pages, qs = _setup("damp", 7, 3)
    qb = make_state(w)
    upload(qb, perm, pages)
    x = W.step_inputs(w, 0)
    xd = {k: v.cuda() for k, v in x.items()}
    o1 = qb.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], seed=3, step=8)
    o2 = torch.empty(1, 7, 3, 128, device="cuda")
    B.stq_prefill(qs.state, xd["q"][None].contiguous(), xd["k"][None].contiguous(), xd["v"][None].contiguous(),
                  xd["alpha"][None].contiguous(), xd["beta"][None].contiguous(), o2, None, seed=3, step=8)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2[0])
    assert torch.equal(qb.pages(), qs.pages())


def test_bounded_wait_times_out_and_writes_nothing():
    w, fmt, perm, pages, qs = _setup("stepquant6", 6, 5)
    L = 4
    x = _prompt(w, L)
    xd = {k: v.cuda() for k, v in x.items()}
    o = torch.full((L, 6, 5, 128), 7.0, device="cuda")
    B.stq_set_wait_limit(qs.state, 20_000_000, stall_first_wait=True)
    B.stq_prefill(qs.state, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o, None, step=1)
    assert B.stq_device_status(qs.state, clear=True) == B.STQ_ERR_DEVICE_TIMEOUT
    assert np.array_equal(download(qs), pages)
    assert bool((o == 7.0).all())
    B.stq_set_wait_limit(qs.state, 0, stall_first_wait=False)
    B.stq_prefill(qs.state, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o, None, step=1)
    assert B.stq_device_status(qs.state) == B.STQ_OK
    ref, o_ref, _, margins = _oracle(fmt, perm, pages, w.heads, x, 0, 1)
    assert np.array_equal(o.cpu().numpy().reshape(L, -1, 128), o_ref)
    _check_pages(fmt, download(qs), ref, margins)


@pytest.mark.parametrize("name,L", [("stepquant6", 130), ("stepquant4_kda", 131)])
def test_prompt_longer_than_the_scalar_chunk(name, L):
    # beta and the scalar gate are staged 128 tokens at a time: cross a chunk boundary
    _run(name, 5, 3, L)
