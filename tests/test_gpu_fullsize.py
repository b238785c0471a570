"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times: one stq_decode_step over every page of the batch (256 to
4,096 requests x 32 heads), checked on sampled pages the oracle steps one by
one.

The state is the GPU's own quantization of a device-generated fp32 state,
except at the sampled positions, which hold oracle-made pages (from a small
CPU-generated batch of the same workload) and get CPU-generated step inputs;
the precision map is the oracle's calibration of that small batch.  So every
oracle input and expected value comes from the generators and the oracle, and
the kernel runs the full-size grid with its wrap-around and ragged tail.
Samples: the first and last pages, both sides of the grid-wrap boundaries
for 2 and 3 resident CTAs per SM, and seeded random positions.  Two chained
steps (each side continues from its own result).  Bar: o, row scales and
packed pages bit-identical, code mismatches only inside the rounding band.
The per-window path (stq_window_step) and the prefill (stq_prefill, a
64-token prompt) are checked the same way, the window over one whole
window, its buffer rows included.
"""
import numpy as np
import pytest
import torch

import oracle as O
from linear_attention_recurrent_delta_b200 import binding as B
from linear_attention_recurrent_delta_b200 import workloads as W

from parity_util import BAND, add_counts, assert_plain_ok, check_against_plain, make_state, maps_agree, plain_step

pytestmark = pytest.mark.gpu

SMALL_BATCH = 4   # CPU-generated requests the sampled pages are drawn from


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from linear_attention_recurrent_delta_b200 import build
    build.build()
    B.lib()
    assert torch.cuda.is_available()


def _sample_positions(n, seed):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    pos = {0, 1, n - 2, n - 1}
    for ctas in (2, 3):
        g = sms * ctas
        for m in (1, 2, n // g):
            for d in (-1, 0):
                if 0 <= m * g + d < n:
                    pos.add(m * g + d)
    rng = np.random.default_rng(seed)
    pos.update(int(x) for x in rng.integers(0, n, 12))
    return sorted(pos)


@pytest.mark.parametrize("index", [1, 2, 3, 4])
def test_full_size_step_on_sampled_pages(index):
    w = W.WORKLOADS[index]
    H, n = w.heads, w.pages
    fmt = O.format_from_spec(w.format)

    # oracle side: map and pages of a small CPU-generated batch
    S_small = W.initial_state(w, batch=SMALL_BATCH).numpy()
    perm = O.rank_rows(fmt, S_small)
    pos = _sample_positions(n, w.seed)
    src = [(i % SMALL_BATCH, p % H) for i, p in enumerate(pos)]   # (request, head) of S_small per sample
    pages = [O.quantize_page(fmt, S_small[b, h], perm[h]) for b, h in src]

    # full-size GPU state: device-generated, quantized on the GPU with the oracle's map
    qs = make_state(w)
    qs.perm().copy_(torch.from_numpy(np.ascontiguousarray(perm, np.uint8)))
    S_dev = W.initial_state(w, device="cuda")
    B.stq_quantize_state(qs.state, S_dev)
    del S_dev
    torch.cuda.synchronize()
    dev_pages = qs.pages()
    idx = torch.tensor(pos, dtype=torch.long, device="cuda")
    dev_pages[idx] = torch.from_numpy(np.stack([O.pack_page(fmt, pg) for pg in pages])).cuda()

    seed = W.sr_seed(w)
    o = torch.empty(w.batch, H, 128, device="cuda")
    plain_total = {}
    for step in range(2):
        xd = W.step_inputs(w, step, device="cuda")
        xc = W.step_inputs(w, step, batch=SMALL_BATCH)
        for k in xd:
            flat = xd[k].view(n, -1)
            flat[idx] = torch.stack([xc[k][b, h].reshape(-1) for b, h in src]).cuda()
        qs.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o=o, seed=seed, step=step)
        assert B.stq_device_status(qs.state) == B.STQ_OK
        got_o = o.view(n, 128)[idx].cpu().numpy()
        torch.cuda.synchronize()
        got_pages = qs.pages()[idx].cpu().numpy()
        band = 0
        for i, (p, (b, h)) in enumerate(zip(pos, src)):
            # against the plain oracle, from the same packed input
            ref = plain_step(fmt, pages[i], perm[h], xc["q"][b, h].numpy(), xc["k"][b, h].numpy(),
                             xc["v"][b, h].numpy(), xc["alpha"][b, h].numpy(), float(xc["beta"][b, h]),
                             seed, step, p // H, p % H)
            res = check_against_plain(fmt, O.unpack_page(fmt, got_pages[i]), got_o[i], ref, perm[h])
            assert_plain_ok(res, (w.name, step, p))
            add_counts(plain_total, res)
            # the oracle steps its own page in place (each side continues from its own result)
            o_ref, _, margin = O.step_f32(fmt, pages[i], perm[h], xc["q"][b, h].numpy(), xc["k"][b, h].numpy(),
                                          xc["v"][b, h].numpy(), xc["alpha"][b, h].numpy(),
                                          float(xc["beta"][b, h]), seed=seed, step=step, b=p // H, h=p % H,
                                          want_margin=True)
            assert np.array_equal(got_o[i], o_ref), "o of page %d (step %d)" % (p, step)
            if not np.array_equal(got_pages[i], O.pack_page(fmt, pages[i])):
                pg = O.unpack_page(fmt, got_pages[i])
                assert np.array_equal(pg.r.view(np.uint32), pages[i].r.view(np.uint32)), "r of page %d" % p
                bad = pg.code != pages[i].code
                assert np.all(margin[bad] < BAND), "codes of page %d outside the rounding band" % p
                band += int(bad.sum())
        assert band == 0, "%d codes inside the rounding band differ (step %d)" % (band, step)
    print("\n%s, %d sampled pages x 2 steps vs the plain oracle: code flips %d (in the 1e-5 band %d, by the "
          "order bound %d), row scales differing %d, max o rel-L2 %.2e, max state rel-L2 %.2e"
          % (w.name, len(pos), plain_total["flips"], plain_total["in_band"], plain_total["by_bound"],
             plain_total["r_diff"], plain_total["o_rel"], plain_total["state_rel"]))


def test_full_size_calibration_map():
    """The precision map of the full int8row batch (256 requests, summed by
    the GPU in chunks of 32) from the CUDA path equals the oracle's (one
    sequential double sum), except at a tie of scores at a group boundary."""
    w = W.WORKLOADS[1]
    S = W.initial_state(w)
    fmt = O.format_from_spec(w.format)
    perm = O.rank_rows(fmt, S.numpy())
    qs = make_state(w)
    B.stq_calibrate(qs.state, S.cuda())
    torch.cuda.synchronize()
    equal, tied = maps_agree(fmt, S.numpy(), qs.perm().cpu().numpy(), perm)
    assert equal + tied == w.heads


@pytest.mark.parametrize("index,window", [(1, 8), (2, 4), (3, 4), (4, 4)])
def test_full_size_window_on_sampled_pages(index, window):
    """A whole window of stq_window_step over the full batch (the launch
    configuration the benchmark times), checked on the same kind of sampled
    pages: o and the buffer rows bit-identical at every step, the committed
    pages bit-identical outside the rounding band."""
    w = W.WORKLOADS[index]
    H, n = w.heads, w.pages
    fmt = O.format_from_spec(w.format)
    S_small = W.initial_state(w, batch=SMALL_BATCH).numpy()
    perm = O.rank_rows(fmt, S_small)
    pos = _sample_positions(n, w.seed + 1)
    src = [(i % SMALL_BATCH, p % H) for i, p in enumerate(pos)]
    pages = [O.quantize_page(fmt, S_small[b, h], perm[h]) for b, h in src]

    qs = make_state(w)
    qs.perm().copy_(torch.from_numpy(np.ascontiguousarray(perm, np.uint8)))
    S_dev = W.initial_state(w, device="cuda")
    B.stq_quantize_state(qs.state, S_dev)
    del S_dev
    torch.cuda.synchronize()
    idx = torch.tensor(pos, dtype=torch.long, device="cuda")
    qs.pages()[idx] = torch.from_numpy(np.stack([O.pack_page(fmt, pg) for pg in pages])).cuda()
    nbuf = B.stq_window_buffer_bytes(qs.state, window)
    buf = torch.full((nbuf,), 0xFF, dtype=torch.uint8, device="cuda")
    rows = buf.view(torch.float32).view(n, 1 + 2 * window, 128)
    Pb = [np.ones(128, np.float32) for _ in pos]
    Kb = [np.zeros((window, 128), np.float32) for _ in pos]
    Db = [np.zeros((window, 128), np.float32) for _ in pos]

    seed = W.sr_seed(w)
    o = torch.empty(w.batch, H, 128, device="cuda")
    for t in range(window):
        commit = t == window - 1
        xd = W.step_inputs(w, 20 + t, device="cuda")
        xc = W.step_inputs(w, 20 + t, batch=SMALL_BATCH)
        for k in xd:
            flat = xd[k].view(n, -1)
            flat[idx] = torch.stack([xc[k][b, h].reshape(-1) for b, h in src]).cuda()
        B.stq_window_step(qs.state, buf, window, t, commit, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o,
                          seed=seed, step=t)
        assert B.stq_device_status(qs.state) == B.STQ_OK
        got_o = o.view(n, 128)[idx].cpu().numpy()
        got_rows = rows[idx].cpu().numpy()
        torch.cuda.synchronize()
        got_pages = qs.pages()[idx].cpu().numpy()
        for i, (p, (b, h)) in enumerate(zip(pos, src)):
            o_ref, margin = O.window_step_f32(fmt, pages[i], perm[h], Pb[i], Kb[i], Db[i], t, commit,
                                              xc["q"][b, h].numpy(), xc["k"][b, h].numpy(), xc["v"][b, h].numpy(),
                                              xc["alpha"][b, h].numpy(), float(xc["beta"][b, h]), seed=seed, step=t,
                                              b=p // H, h=p % H, want_margin=commit)
            assert np.array_equal(got_o[i], o_ref), "o of page %d (t %d)" % (p, t)
            if not commit:
                assert np.array_equal(got_rows[i][0], Pb[i]), "P of page %d (t %d)" % (p, t)
                assert np.array_equal(got_rows[i][1:2 + t], Kb[i][:t + 1]), "K of page %d (t %d)" % (p, t)
                assert np.array_equal(got_rows[i][1 + window:2 + window + t], Db[i][:t + 1]), "D of page %d" % p
            elif not np.array_equal(got_pages[i], O.pack_page(fmt, pages[i])):
                pg = O.unpack_page(fmt, got_pages[i])
                assert np.array_equal(pg.r.view(np.uint32), pages[i].r.view(np.uint32)), "r of page %d" % p
                bad = pg.code != pages[i].code
                assert np.all(margin[bad] < BAND), "codes of page %d outside the rounding band" % p


def test_full_size_prefill_on_sampled_pages():
    """stq_prefill of a 64-token prompt over the full default batch (the
    benchmark's launch configuration), checked on sampled pages: o of every
    token and the fp32 state bit-identical, pages bit-identical outside the
    rounding band."""
    w = W.WORKLOADS[1]
    H, n, L = w.heads, w.pages, 64
    fmt = O.format_from_spec(w.format)
    S_small = W.initial_state(w, batch=SMALL_BATCH).numpy()
    perm = O.rank_rows(fmt, S_small)
    pos = _sample_positions(n, w.seed + 2)
    src = [(i % SMALL_BATCH, p % H) for i, p in enumerate(pos)]
    pages = [O.quantize_page(fmt, S_small[b, h], perm[h]) for b, h in src]

    qs = make_state(w)
    qs.perm().copy_(torch.from_numpy(np.ascontiguousarray(perm, np.uint8)))
    S_dev = W.initial_state(w, device="cuda")
    B.stq_quantize_state(qs.state, S_dev)
    del S_dev
    torch.cuda.synchronize()
    idx = torch.tensor(pos, dtype=torch.long, device="cuda")
    qs.pages()[idx] = torch.from_numpy(np.stack([O.pack_page(fmt, pg) for pg in pages])).cuda()

    xd = {k: torch.stack([W.step_inputs(w, 40 + l, device="cuda")[k] for l in range(L)]).contiguous()
          for k in ("q", "k", "v", "alpha", "beta")}
    xc = [W.step_inputs(w, 40 + l, batch=SMALL_BATCH) for l in range(L)]
    for k in xd:
        flat = xd[k].view(L, n, -1)
        flat[:, idx] = torch.stack([torch.stack([xc[l][k][b, h].reshape(-1) for b, h in src]) for l in range(L)]).cuda()
    seed = W.sr_seed(w)
    o = torch.empty(L, w.batch, H, 128, device="cuda")
    S_out = torch.empty(w.batch, H, 128, 128, device="cuda")
    B.stq_prefill(qs.state, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o, S_out, seed=seed, step=3)
    assert B.stq_device_status(qs.state) == B.STQ_OK
    got_o = o.view(L, n, 128)[:, idx].cpu().numpy()
    got_S = S_out.view(n, 128, 128)[idx].cpu().numpy()
    torch.cuda.synchronize()
    got_pages = qs.pages()[idx].cpu().numpy()
    for i, (p, (b, h)) in enumerate(zip(pos, src)):
        arr = {k: np.stack([xc[l][k][b, h].numpy().reshape(-1) for l in range(L)]) for k in xd}
        o_ref, tp, margin = O.prefill_f32(fmt, pages[i], perm[h], arr["q"], arr["k"], arr["v"], arr["alpha"],
                                          arr["beta"][:, 0], seed=seed, step=3, b=p // H, h=p % H, want_tp=True,
                                          want_margin=True)
        assert np.array_equal(got_o[:, i], o_ref), "o of page %d" % p
        S_ref = np.zeros((128, 128), np.float32)
        c = pages[i].c if fmt.col_scales else np.ones(128, np.float32)
        S_ref[perm[h]] = tp * c[None, :]
        assert np.array_equal(got_S[i], S_ref), "state of page %d" % p
        if not np.array_equal(got_pages[i], O.pack_page(fmt, pages[i])):
            pg = O.unpack_page(fmt, got_pages[i])
            assert np.array_equal(pg.r.view(np.uint32), pages[i].r.view(np.uint32)), "r of page %d" % p
            bad = pg.code != pages[i].code
            assert np.all(margin[bad] < BAND), "codes of page %d outside the rounding band" % p
