"""GPU parity of the per-window decode step (stq_window_step) with the oracle.

Both sides start each window from the same packed pages.  A step that does
not commit must match bit for bit: o, the buffer rows it defines (P, K[0..t],
D[0..t]) and the pages, which it must leave unchanged.  A committing step
must match o bit for bit and the requantized pages bit for bit, except codes
whose pre-rounding value the oracle reports within 1e-5 (relative) of a
rounding boundary.  The device buffer starts as 0xFF bytes (NaN floats): a
window's first step reads none of it.
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


def _setup(name, batch, heads):
    base = [w for w in W.WORKLOADS if w.fmt == name and w.index > 0][0]
    w = W.Workload(base.index, base.name, name, batch, heads, 2, base.gate_mu, base.gate_sigma, base.seed)
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    qs = make_state(w)
    upload(qs, perm, pages)
    return w, fmt, perm, pages, qs


class OracleWindow:
    """The oracle's side: unpacked pages and a buffer per page."""

    def __init__(self, fmt, perm, pages, heads, window):
        self.fmt, self.perm, self.H, self.W = fmt, perm, heads, window
        n = len(pages)
        self.pages = [O.unpack_page(fmt, pages[i]) for i in range(n)]
        self.P = np.ones((n, 128), np.float32)
        self.K = np.zeros((n, window, 128), np.float32)
        self.D = np.zeros((n, window, 128), np.float32)

    def step(self, x, t, commit, seed, step):
        n = len(self.pages)
        arr = {k: v.numpy().reshape(n, -1) for k, v in x.items()}
        o = np.zeros((n, 128), np.float32)
        margins = []
        for i in range(n):
            b, h = divmod(i, self.H)
            o[i], mg = O.window_step_f32(self.fmt, self.pages[i], self.perm[h], self.P[i], self.K[i], self.D[i], t,
                                         commit, arr["q"][i], arr["k"][i], arr["v"][i], arr["alpha"][i],
                                         float(arr["beta"][i][0]), seed=seed, step=step, b=b, h=h,
                                         want_margin=commit)
            margins.append(mg)
        return o, margins

    def packed(self):
        return np.stack([O.pack_page(self.fmt, p) for p in self.pages])


def _gpu_buffer(qs, window):
    n = B.stq_window_buffer_bytes(qs.state, window)
    assert n == qs.batch * qs.heads * 512 * (1 + 2 * window)
    return torch.full((n,), 0xFF, dtype=torch.uint8, device="cuda")


def _buffer_rows(buf, n_pages, window):
    f = buf.view(torch.float32).view(n_pages, 1 + 2 * window, 128).cpu().numpy()
    return f[:, 0], f[:, 1:1 + window], f[:, 1 + window:]


def _check_commit(fmt, got, ref, margins):
    mism = band = 0
    for i in range(len(ref)):
        if np.array_equal(got[i], ref[i]):
            continue
        pg, pe = O.unpack_page(fmt, got[i]), O.unpack_page(fmt, ref[i])
        assert np.array_equal(pg.r.view(np.uint32), pe.r.view(np.uint32)), i
        bad = pg.code != pe.code
        mism += int(bad.sum())
        band += int(np.sum(bad & (margins[i] < BAND)))
        assert np.abs(pg.code[bad] - pe.code[bad]).max() <= 1
    assert mism == band, (mism, band)
    return mism


def _run_windows(name, batch, heads, window, windows, commit_at=None, seed_steps=0):
    w, fmt, perm, pages, qs = _setup(name, batch, heads)
    n = batch * heads
    seed = W.sr_seed(w)
    buf = _gpu_buffer(qs, window)
    step = seed_steps
    band_total = 0
    for wi in range(windows):
        orc = OracleWindow(fmt, perm, pages, heads, window)
        last = window - 1 if commit_at is None else commit_at[wi]
        for t in range(last + 1):
            commit = t == last
            x = W.step_inputs(w, step)
            xd = {k: v.cuda() for k, v in x.items()}
            o = torch.empty(batch, heads, 128, device="cuda")
            B.stq_window_step(qs.state, buf, window, t, commit, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"],
                              o, seed=seed, step=step)
            o_ref, margins = orc.step(x, t, commit, seed, step)
            assert B.stq_device_status(qs.state) == B.STQ_OK, (wi, t)
            assert np.array_equal(o.cpu().numpy().reshape(n, 128), o_ref), (wi, t)
            got = download(qs)
            if not commit:
                assert np.array_equal(got, pages), (wi, t)          # pages fixed within a window
                Pg, Kg, Dg = _buffer_rows(buf, n, window)
                assert np.array_equal(Pg, orc.P), (wi, t)
                assert np.array_equal(Kg[:, :t + 1], orc.K[:, :t + 1]), (wi, t)
                assert np.array_equal(Dg[:, :t + 1], orc.D[:, :t + 1]), (wi, t)
            else:
                ref = orc.packed()
                band_total += _check_commit(fmt, got, ref, margins)
                pages = ref
                upload(qs, perm, pages)      # the next window starts from the oracle's pages on both sides
            step += 1
    return band_total


@pytest.mark.parametrize("name", ["stepquant6", "int8row", "stepquant4_kda", "damp"])
def test_window_of_four_matches_oracle(name):
    _run_windows(name, batch=9, heads=5, window=4, windows=2)


def test_ring_reuse_many_pages_per_cta():
    # more pages than resident CTAs x ring stages: every stage is refilled several times
    _run_windows("int8row", batch=96, heads=20, window=3, windows=1)


def test_longest_window_and_early_commit():
    _run_windows("stepquant4_kda", batch=5, heads=3, window=B.STQ_WINDOW_MAX, windows=1)
    _run_windows("stepquant6", batch=7, heads=4, window=8, windows=3, commit_at=[2, 0, 7])


def test_window_of_one_is_a_commit_each_step():
    _run_windows("damp", batch=6, heads=5, window=1, windows=3)


@pytest.mark.parametrize("stochastic", [False, True])
def test_runtime_format(stochastic, monkeypatch):
    """A format outside the four compiled-in ones (block widths read at run time)."""
    name = "window_runtime_%d" % stochastic
    spec = {"groups": [(16, "fp16", 0), (32, "int", 7), (48, "int", 5), (32, "int", 2)], "col_scales": True,
            "gate_vector": True, "stochastic": stochastic}
    monkeypatch.setitem(W.FORMATS, name, spec)
    kda = [w for w in W.WORKLOADS if w.fmt == "stepquant4_kda"][0]
    monkeypatch.setattr(W, "WORKLOADS", list(W.WORKLOADS) + [
        W.Workload(kda.index, name, name, 6, 4, 2, kda.gate_mu, kda.gate_sigma, kda.seed + 7)])
    _run_windows(name, batch=6, heads=4, window=3, windows=2)


def test_window_against_plain_steps_from_the_same_page():
    """Within a window the outputs follow the exact rule from the page; the
    per-step path requantizes every step.  Both stay within the per-step
    path's quantization error of each other (rel-L2 of o below 5e-2)."""
    w, fmt, perm, pages, qs = _setup("int8row", 8, 4)
    qb = make_state(w)
    upload(qb, perm, pages)
    buf = _gpu_buffer(qs, 8)
    for t in range(8):
        x = W.step_inputs(w, t)
        xd = {k: v.cuda() for k, v in x.items()}
        o_w = torch.empty(8, 4, 128, device="cuda")
        B.stq_window_step(qs.state, buf, 8, t, t == 7, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o_w,
                          step=t)
        o_p = qb.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], step=t)
        rel = float(torch.linalg.norm(o_w - o_p) / torch.linalg.norm(o_p))
        assert rel < 5e-2, (t, rel)


@pytest.mark.parametrize("commit", [False, True])
def test_bounded_wait_times_out_and_writes_nothing(commit):
    """The test hook makes every CTA's first wait run out (20 ms): the status
    word reports it, no page, buffer row or o is written, and the next step
    runs normally and matches the oracle."""
    w, fmt, perm, pages, qs = _setup("stepquant6", 6, 5)
    n = w.batch * w.heads
    window, t = 4, (3 if commit else 0)
    buf = _gpu_buffer(qs, window)
    x = W.step_inputs(w, 0)
    xd = {k: v.cuda() for k, v in x.items()}
    o = torch.full((w.batch, w.heads, 128), 7.0, device="cuda")
    if commit:   # a committing step needs a window so far: steps 0 .. 2 first
        orc = OracleWindow(fmt, perm, pages, w.heads, window)
        for s in range(3):
            xs = W.step_inputs(w, 10 + s)
            xsd = {k: v.cuda() for k, v in xs.items()}
            B.stq_window_step(qs.state, buf, window, s, False, xsd["q"], xsd["k"], xsd["v"], xsd["alpha"],
                              xsd["beta"], o, step=s)
            orc.step(xs, s, False, 0, s)
        o.fill_(7.0)
    before = buf.clone()
    B.stq_set_wait_limit(qs.state, 20_000_000, stall_first_wait=True)
    B.stq_window_step(qs.state, buf, window, t, commit, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o,
                      step=t)
    assert B.stq_device_status(qs.state, clear=True) == B.STQ_ERR_DEVICE_TIMEOUT
    assert np.array_equal(download(qs), pages)
    assert torch.equal(buf, before)
    assert bool((o == 7.0).all())
    B.stq_set_wait_limit(qs.state, 0, stall_first_wait=False)
    B.stq_window_step(qs.state, buf, window, t, commit, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o,
                      step=t)
    assert B.stq_device_status(qs.state) == B.STQ_OK
    if not commit:
        orc = OracleWindow(fmt, perm, pages, w.heads, window)
    o_ref, margins = orc.step(x, t, commit, 0, t)
    assert np.array_equal(o.cpu().numpy().reshape(n, 128), o_ref)
    if commit:
        _check_commit(fmt, download(qs), orc.packed(), margins)
