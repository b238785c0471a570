"""GPU parity of the paged step (stq_decode_step_slots) and of request copy-out.

Input row i steps the pages of the request in state slot table[i]; the
oracle steps the same pages from the same packed input with row i's inputs
and the slot as the request index of the stochastic-rounding counter.  Pages
of slots not in the table must not change at all.  A slot outside the state
is caught on the device: its pages are neither read nor written, its o row is
NaN, and the status reports an invalid argument.
"""
import numpy as np
import pytest
import torch

import oracle as O
from linear_attention_recurrent_delta_b200 import binding as B
from linear_attention_recurrent_delta_b200 import workloads as W

from parity_util import download, make_state, oracle_quantize, oracle_step, upload

pytestmark = pytest.mark.gpu

STATE_BATCH, HEADS = 9, 5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from linear_attention_recurrent_delta_b200 import build
    build.build()
    B.lib()
    assert torch.cuda.is_available()


def _setup(name):
    base = [w for w in W.WORKLOADS if w.fmt == name and w.index > 0][0]
    w = base.resized(batch=STATE_BATCH, heads=HEADS, steps=2)
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    qs = make_state(w)
    upload(qs, perm, pages)
    return w, fmt, perm, pages, qs


def _oracle_slots(fmt, perm, pages, table, x, seed, step):
    """Oracle: row i steps the pages of slot table[i]; returns (pages', o[rows, H, 128])."""
    out = pages.copy()
    o = np.zeros((len(table), HEADS, 128), np.float32)
    for i, slot in enumerate(table):
        for h in range(HEADS):
            pg = O.unpack_page(fmt, out[slot * HEADS + h])
            o[i, h], _, _ = O.step_f32(fmt, pg, perm[h], x["q"][i, h].numpy(), x["k"][i, h].numpy(),
                                       x["v"][i, h].numpy(), x["alpha"][i, h].numpy(), float(x["beta"][i, h]),
                                       seed=seed, step=step, b=slot, h=h)
            out[slot * HEADS + h] = O.pack_page(fmt, pg)
    return out, o


def _step_slots(qs, table, x, seed, step):
    xd = {k: v.cuda() for k, v in x.items()}
    t = torch.tensor(table, dtype=torch.int32, device="cuda")
    o = torch.empty(len(table), HEADS, 128, device="cuda")
    B.stq_decode_step_slots(qs.state, t, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o, seed=seed,
                            step=step)
    return o


@pytest.mark.parametrize("name", ["stepquant6", "int8row", "stepquant4_kda", "damp"])
def test_slot_subset_matches_oracle_and_leaves_other_pages(name):
    w, fmt, perm, pages, qs = _setup(name)
    seed = W.sr_seed(w)
    table = [7, 2, 5, 0]
    for step in range(2):
        x = W.step_inputs(w.resized(batch=len(table)), step)
        o = _step_slots(qs, table, x, seed, step)
        assert B.stq_device_status(qs.state) == B.STQ_OK
        expect, o_ref = _oracle_slots(fmt, perm, pages, table, x, seed, step)
        got = download(qs)
        assert np.array_equal(o.cpu().numpy(), o_ref)
        assert np.array_equal(got, expect)          # stepped pages match, all others unchanged
        pages = expect


def test_identity_table_equals_the_plain_step():
    w, fmt, perm, pages, qs = _setup("damp")
    qb = make_state(w)
    upload(qb, perm, pages)
    x = W.step_inputs(w, 0)
    xd = {k: v.cuda() for k, v in x.items()}
    o_plain = qb.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], seed=11, step=3)
    o_slots = _step_slots(qs, list(range(STATE_BATCH)), x, 11, 3)
    torch.cuda.synchronize()
    assert torch.equal(o_plain, o_slots)
    assert torch.equal(qb.pages(), qs.pages())


def test_out_of_range_slot_is_reported_and_touches_nothing():
    w, fmt, perm, pages, qs = _setup("stepquant6")
    before = qs.view.clone()
    table = [3, STATE_BATCH + 90, 1]
    x = W.step_inputs(w.resized(batch=len(table)), 0)
    o = _step_slots(qs, table, x, 5, 0)
    assert B.stq_device_status(qs.state, clear=True) == B.STQ_ERR_INVALID_ARG
    assert torch.isnan(o[1]).all()
    good = [3, 1]
    xg = {k: v[[0, 2]].contiguous() for k, v in x.items()}
    expect, o_ref = _oracle_slots(fmt, perm, pages, good, xg, 5, 0)
    assert np.array_equal(o[[0, 2]].cpu().numpy(), o_ref)
    assert np.array_equal(download(qs), expect)     # the two good requests stepped, nothing else written
    L = qs.layout
    hdr = slice(0, L["pages_offset"])
    assert torch.equal(qs.view[hdr][4:], before[hdr][4:])   # map and header untouched (status word aside)
    assert B.stq_device_status(qs.state) == B.STQ_OK        # cleared


def test_request_copy_out_and_back_restores_it():
    w, fmt, perm, pages, qs = _setup("stepquant4_kda")
    off, nbytes = B.stq_request_pages(qs.state, 4)
    saved = qs.view[off:off + nbytes].clone()
    x = W.step_inputs(w, 0)
    xd = {k: v.cuda() for k, v in x.items()}
    qs.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"])
    torch.cuda.synchronize()
    assert not torch.equal(qs.view[off:off + nbytes], saved)
    qs.view[off:off + nbytes].copy_(saved)          # a plain device copy restores request 4
    got = download(qs)
    assert np.array_equal(got[4 * HEADS:5 * HEADS], pages[4 * HEADS:5 * HEADS])


@pytest.mark.parametrize("name", ["stepquant6", "int8row", "stepquant4_kda", "damp"])
def test_many_pages_per_cta_with_a_bad_slot(name):
    """More work than the persistent grid holds at once (800 requests x 4
    heads: every CTA refills its ring several times, so the slots of later
    items are resolved inside the page loop), a random permutation of the
    slots, and one row near the end naming a slot outside the state.  The
    oracle steps every page with its row's inputs in slot order; the pages
    of the slot the bad row displaced stay as they were."""
    base = [w for w in W.WORKLOADS if w.fmt == name and w.index > 0][0]
    w = base.resized(batch=800, heads=4, steps=2)
    H = w.heads
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    qs = make_state(w)
    upload(qs, perm, pages)
    rng = np.random.default_rng(5)
    table = rng.permutation(w.batch).astype(np.int32)
    bad_row = 700                      # item 2,800: past the first ring fill of every CTA
    dropped = int(table[bad_row])
    table[bad_row] = w.batch + 17
    x = W.step_inputs(w, 0)
    seed = W.sr_seed(w)
    xd = {k: v.cuda() for k, v in x.items()}
    o = torch.empty(w.batch, H, 128, device="cuda")
    B.stq_decode_step_slots(qs.state, torch.from_numpy(table).cuda(), xd["q"], xd["k"], xd["v"], xd["alpha"],
                            xd["beta"], o, seed=seed, step=1)
    assert B.stq_device_status(qs.state, clear=True) == B.STQ_ERR_INVALID_ARG
    good = np.array([i for i in range(w.batch) if i != bad_row])
    xs = {k: torch.zeros_like(v) for k, v in x.items()}
    for k in x:
        xs[k][torch.from_numpy(table[good]).long()] = x[k][torch.from_numpy(good)]
    expect, o_ref = oracle_step(fmt, w, w.batch, H, pages, perm, xs, seed, 1)
    expect[dropped * H:(dropped + 1) * H] = pages[dropped * H:(dropped + 1) * H]
    got = download(qs)
    o = o.cpu().numpy()
    assert np.isnan(o[bad_row]).all()
    assert np.array_equal(o[good], o_ref.reshape(w.batch, H, 128)[table[good]])
    assert np.array_equal(got, expect)


@pytest.mark.parametrize("stochastic", [False, True])
def test_runtime_format(stochastic, monkeypatch):
    """A format outside the four compiled-in ones (block widths read at run
    time) through the slot table, many pages per CTA."""
    name = "slots_runtime_%d" % stochastic
    spec = {"groups": [(32, "int", 7), (16, "fp16", 0), (48, "int", 5), (32, "int", 2)], "col_scales": True,
            "gate_vector": True, "stochastic": stochastic}
    monkeypatch.setitem(W.FORMATS, name, spec)
    kda = [w for w in W.WORKLOADS if w.fmt == "stepquant4_kda" and w.index > 0][0]
    w = W.Workload(kda.index, name, name, 400, 4, 2, kda.gate_mu, kda.gate_sigma, kda.seed + 13)
    H = w.heads
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    qs = make_state(w)
    upload(qs, perm, pages)
    table = np.random.default_rng(8).permutation(w.batch).astype(np.int32)
    x = W.step_inputs(w, 0)
    seed = W.sr_seed(w)
    xd = {k: v.cuda() for k, v in x.items()}
    o = torch.empty(w.batch, H, 128, device="cuda")
    B.stq_decode_step_slots(qs.state, torch.from_numpy(table).cuda(), xd["q"], xd["k"], xd["v"], xd["alpha"],
                            xd["beta"], o, seed=seed, step=2)
    assert B.stq_device_status(qs.state) == B.STQ_OK
    xs = {k: torch.zeros_like(v) for k, v in x.items()}
    for k in x:
        xs[k][torch.from_numpy(table).long()] = x[k]
    expect, o_ref = oracle_step(fmt, w, w.batch, H, pages, perm, xs, seed, 2)
    assert np.array_equal(o.cpu().numpy(), o_ref.reshape(w.batch, H, 128)[table])
    assert np.array_equal(download(qs), expect)
