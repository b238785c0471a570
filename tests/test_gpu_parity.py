"""GPU parity: the CUDA path through the C ABI against the CPU oracle, element
by element, on the same seeded inputs.

Sizes: every format at B x H = 37 x 9 = 333 pages (more pages than resident
CTAs, so the persistent grid wraps with a ragged tail), and the tiny GDN
workload (1 x 4 pages) over its full 64-step trajectory.  The bar:
o and the dequantized state within rel-L2 1e-5, integer codes and packed words
bit-identical except elements whose pre-rounding value lies within 1e-5 of a
rounding boundary (counted), row scales bit-identical; the free-running
64-step o within rel-L2 1e-3.  The kernels reproduce the oracle's canonical
fp32 evaluation, so the expected mismatch count is zero.
"""
import numpy as np
import pytest
import torch

import oracle as O
from linear_attention_recurrent_delta_b200 import binding as B
from linear_attention_recurrent_delta_b200 import workloads as W

from parity_util import (add_counts, assert_plain_ok, check_against_plain, compare_pages, download, make_state,
                         maps_agree, oracle_quantize, oracle_step, plain_step, rel_l2, step_inputs_gpu, upload)

pytestmark = pytest.mark.gpu

NAMES = list(W.FORMATS)


def _small(name, batch=37, heads=9, steps=4):
    w = [x for x in W.WORKLOADS if x.fmt == name and x.index > 0][0]
    return w.resized(batch=batch, heads=heads, steps=steps)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from linear_attention_recurrent_delta_b200 import build
    build.build()
    B.lib()
    assert torch.cuda.is_available()


@pytest.mark.parametrize("name", NAMES)
def test_calibrate_and_quantize_match_oracle(name):
    w = _small(name)
    S = W.initial_state(w)
    fmt, perm, pages = oracle_quantize(w, S.numpy())
    qs = make_state(w)
    qs.calibrate_and_quantize(S.cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(qs.perm().cpu().numpy(), perm)
    res = compare_pages(fmt, download(qs), pages)
    assert res["pages_equal"] == res["pages"], res


@pytest.mark.parametrize("name", NAMES)
def test_dequantize_matches_oracle(name):
    w = _small(name)
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    qs = make_state(w)
    upload(qs, perm, pages)
    got = qs.dequantize().cpu().numpy()
    for i in range(w.pages):
        b, h = divmod(i, w.heads)
        expect = O.dequantize_page(fmt, O.unpack_page(fmt, pages[i]), perm[h])
        np.testing.assert_array_equal(got[b, h], expect)


@pytest.mark.parametrize("name", NAMES)
def test_step_matches_oracle_from_the_same_input(name):
    w = _small(name)
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    qs = make_state(w)
    seed = W.sr_seed(w)
    for step in range(w.steps):
        x, xd = step_inputs_gpu(w, step)
        upload(qs, perm, pages)
        o_gpu = qs.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], seed=seed, step=step)
        got = download(qs)
        expect, o_ref = oracle_step(fmt, w, w.batch, w.heads, pages, perm, x, seed, step)
        o_gpu = o_gpu.cpu().numpy().reshape(w.pages, 128)
        assert rel_l2(o_gpu, o_ref) <= 1e-5
        assert np.array_equal(o_gpu, o_ref), "o differs bitwise in %d elements" % np.sum(o_gpu != o_ref)
        res = compare_pages(fmt, got, expect, perm, (pages, x, seed, step, w.heads))
        assert res["code_mismatch"] == res["band_mismatch"], res
        assert res["r_mismatch"] == 0, res
        assert res["pages_equal"] == res["pages"], res
        # dequantized states agree too
        qs_deq = qs.dequantize().cpu().numpy()
        for i in (0, w.pages // 2, w.pages - 1):
            b, h = divmod(i, w.heads)
            ref = O.dequantize_page(fmt, O.unpack_page(fmt, expect[i]), perm[h])
            assert rel_l2(qs_deq[b, h], ref) <= 1e-5
        pages = expect


@pytest.mark.parametrize("name", NAMES)
def test_step_within_the_plain_oracle_band(name):
    """The same steps against the oracle's plain evaluation (every column sum
    one fma chain over the key channels in natural order): o and the
    dequantized state within rel-L2 1e-5; codes and row scales identical
    except inside the 1e-5 band or the fp32 bound of any summation order
    around a rounding boundary; the flips are counted and printed."""
    w = _small(name)
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    qs = make_state(w)
    seed = W.sr_seed(w)
    total = {}
    for step in range(w.steps):
        x, xd = step_inputs_gpu(w, step)
        upload(qs, perm, pages)
        o_gpu = qs.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], seed=seed, step=step)
        got = download(qs)
        o_gpu = o_gpu.cpu().numpy().reshape(w.pages, 128)
        xs = {k: v.numpy().reshape(w.pages, -1) for k, v in x.items()}
        for i in range(w.pages):
            b, h = divmod(i, w.heads)
            ref = plain_step(fmt, O.unpack_page(fmt, pages[i]), perm[h], xs["q"][i], xs["k"][i], xs["v"][i],
                             xs["alpha"][i], float(xs["beta"][i][0]), seed, step, b, h)
            res = check_against_plain(fmt, O.unpack_page(fmt, got[i]), o_gpu[i], ref, perm[h])
            assert_plain_ok(res, (name, step, i))
            add_counts(total, res)
        pages = got
    print("\n%s vs the plain oracle, %d page-steps: code flips %d (in the 1e-5 band %d, by the order bound %d), "
          "row scales differing %d, max o rel-L2 %.2e, max state rel-L2 %.2e"
          % (name, w.pages * w.steps, total["flips"], total["in_band"], total["by_bound"], total["r_diff"],
             total["o_rel"], total["state_rel"]))


def test_tiny_trajectory_free_running():
    """Workload 0 (1 x 4 pages, 64 steps): GPU and oracle each run free from
    their own quantization of the same fp32 state."""
    w = W.WORKLOADS[0]
    S = W.initial_state(w)
    fmt, perm, pages = oracle_quantize(w, S.numpy())
    qs = make_state(w)
    qs.calibrate_and_quantize(S.cuda())
    seed = W.sr_seed(w)
    worst, exact = 0.0, 0
    for step in range(w.steps):
        x, xd = step_inputs_gpu(w, step)
        o_gpu = qs.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], seed=seed, step=step)
        pages, o_ref = oracle_step(fmt, w, w.batch, w.heads, pages, perm, x, seed, step)
        o_gpu = o_gpu.cpu().numpy().reshape(w.pages, 128)
        worst = max(worst, rel_l2(o_gpu, o_ref))
        exact += int(np.array_equal(o_gpu, o_ref))
        assert rel_l2(o_gpu, o_ref) <= 1e-3, step
    assert np.array_equal(download(qs), pages)
    print("trajectory: worst rel-L2 %.3g, bit-identical o on %d/%d steps" % (worst, exact, w.steps))


@pytest.mark.parametrize("name", ["int8row", "stepquant4_kda", "damp"])
def test_long_trajectory_other_formats(name):
    """Free-running trajectories of the other formats at a small batch, over
    their workload's step count and at least 64 steps (the uniform INT8
    workload runs 128)."""
    full = [x for x in W.WORKLOADS if x.fmt == name and x.index > 0][0]
    w = _small(name, batch=3, heads=4, steps=max(64, full.steps))
    S = W.initial_state(w)
    fmt, perm, pages = oracle_quantize(w, S.numpy())
    qs = make_state(w)
    qs.calibrate_and_quantize(S.cuda())
    seed = W.sr_seed(w)
    for step in range(w.steps):
        x, xd = step_inputs_gpu(w, step)
        o_gpu = qs.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], seed=seed, step=step)
        pages, o_ref = oracle_step(fmt, w, w.batch, w.heads, pages, perm, x, seed, step)
        assert rel_l2(o_gpu.cpu().numpy().reshape(w.pages, 128), o_ref) <= 1e-3, step
    assert np.array_equal(download(qs), pages)


@pytest.mark.parametrize("name", ["stepquant6", "int8row", "stepquant4_kda"])
def test_identity_step_keeps_codes_on_gpu(name):
    w = _small(name, batch=5, heads=3)
    S = W.initial_state(w)
    qs = make_state(w)
    qs.calibrate_and_quantize(S.cuda())
    before = download(qs)
    fmt = O.format_from_spec(w.format)
    x, xd = step_inputs_gpu(w, 0)
    ones = torch.ones_like(xd["alpha"])
    zeros = torch.zeros_like(xd["beta"])
    qs.step(xd["q"], xd["k"], xd["v"], ones, zeros)
    after = download(qs)
    for i in range(w.pages):
        pa, pb = O.unpack_page(fmt, after[i]), O.unpack_page(fmt, before[i])
        np.testing.assert_array_equal(pa.code, pb.code)
        assert np.all(np.abs(pa.r - pb.r) <= np.spacing(pb.r))


def test_zero_state_and_zero_rows():
    w = _small("stepquant6", batch=2, heads=3, steps=2)
    S = W.initial_state(w)
    S[0] = 0.0           # request 0: an all-zero state
    S[1, 1, 7] = 0.0     # one zero key row
    S[1, 2, :, 5] = 0.0  # one zero value column
    fmt, perm, pages = oracle_quantize(w, S.numpy())
    qs = make_state(w)
    qs.calibrate_and_quantize(S.cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(qs.perm().cpu().numpy(), perm)
    assert np.array_equal(download(qs), pages)
    seed = W.sr_seed(w)
    for step in range(2):
        x, xd = step_inputs_gpu(w, step)
        o_gpu = qs.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], seed=seed, step=step)
        pages, o_ref = oracle_step(fmt, w, w.batch, w.heads, pages, perm, x, seed, step)
        assert np.array_equal(o_gpu.cpu().numpy().reshape(w.pages, 128), o_ref)
        assert np.array_equal(download(qs), pages)


def test_non_finite_input_does_not_fault_and_stays_local():
    w = _small("damp", batch=2, heads=2, steps=1)
    S = W.initial_state(w)
    fmt, perm, pages = oracle_quantize(w, S.numpy())
    qs = make_state(w)
    upload(qs, perm, pages)
    x, xd = step_inputs_gpu(w, 0)
    xd["v"][0, 0, 3] = float("nan")
    xd["q"][1, 1, 0] = float("inf")
    o = qs.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], seed=1, step=0)
    assert B.stq_device_status(qs.state) == B.STQ_OK
    x["v"][0, 0, 3] = float("nan")
    x["q"][1, 1, 0] = float("inf")
    expect, o_ref = oracle_step(fmt, w, w.batch, w.heads, pages, perm, x, 1, 0)
    got = download(qs)
    # pages 1 and 2 saw only finite inputs: identical; page 3's state is finite (only o is not)
    for i in (1, 2, 3):
        assert np.array_equal(got[i], expect[i])
    np.testing.assert_array_equal(o.cpu().numpy().reshape(4, 128)[1:3], o_ref[1:3])


def test_host_entry_point_matches_device_entry_point():
    w = _small("stepquant6", batch=4, heads=5, steps=1)
    S = W.initial_state(w).cuda()
    qa, qb = make_state(w), make_state(w)
    qa.calibrate_and_quantize(S)
    qb.calibrate_and_quantize(S)
    x, xd = step_inputs_gpu(w, 0)
    o_dev = qa.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], seed=5, step=2)
    host = {k: v.pin_memory() for k, v in x.items()}
    o_host = torch.empty_like(host["q"]).pin_memory()
    io = torch.empty(B.stq_decode_io_bytes(qb.state) + 256, dtype=torch.uint8, device="cuda")
    off = (-io.data_ptr()) % 256
    io = io[off:off + B.stq_decode_io_bytes(qb.state)]
    B.stq_decode_step_host(qb.state, host["q"], host["k"], host["v"], host["alpha"], host["beta"], o_host, io,
                           seed=5, step=2)
    torch.cuda.synchronize()
    assert torch.equal(o_host, o_dev.cpu())
    assert torch.equal(qa.pages(), qb.pages())


DEGENERATE = {
    "full_decay": lambda x: x["alpha"].zero_(),            # A S = 0: T' = beta k (v/c)^T, a rank-1 state
    "decay_only": lambda x: x["beta"].zero_(),             # no delta write: S' = A S
    "zero_key": lambda x: x["k"].zero_(),                  # u = 0 and beta k = 0: S' = A S
    "zero_query": lambda x: x["q"].zero_(),                # o = 0 exactly (+0)
    "zero_value": lambda x: x["v"].zero_(),                # e = -u: pure erasure along k
    "no_decay_full_write": lambda x: (x["alpha"].fill_(1.0), x["beta"].fill_(1.0)),
}


@pytest.mark.parametrize("case", list(DEGENERATE))
@pytest.mark.parametrize("name", ["stepquant6", "stepquant4_kda", "damp"])
def test_degenerate_inputs_match_oracle(name, case):
    """The method's degenerate inputs, GPU against oracle from the same packed
    state: every page and o bit-identical."""
    w = _small(name, batch=3, heads=5, steps=1)
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    qs = make_state(w)
    upload(qs, perm, pages)
    x = W.step_inputs(w, 0)
    DEGENERATE[case](x)
    xd = {k: v.cuda() for k, v in x.items()}
    seed = W.sr_seed(w)
    o = qs.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], seed=seed, step=0)
    expect, o_ref = oracle_step(fmt, w, w.batch, w.heads, pages, perm, x, seed, 0)
    got_o = o.cpu().numpy().reshape(w.pages, 128)
    assert np.array_equal(got_o.view(np.uint32), o_ref.view(np.uint32)), case   # signs of zeros too
    res = compare_pages(fmt, download(qs), expect)
    assert res["pages_equal"] == res["pages"], (case, res)
    if case == "zero_query":
        assert not np.any(got_o.view(np.uint32))


CUSTOM_FORMATS = {
    # widths 7 and 5 (4+2+1 and 4+1 planes), column scales, GDN: the run-time-width kernel
    "custom_int7_int5": {"groups": [(48, "int", 7), (80, "int", 5)],
                         "col_scales": True, "stochastic": False, "gate_vector": False},
    # FP16 rows in the middle of the page, widths 3 and 2, KDA gate, stochastic rounding
    "custom_fp16_int3_int2_sr": {"groups": [(16, "int", 8), (32, "fp16", 0), (48, "int", 3), (32, "int", 2)],
                                 "col_scales": True, "stochastic": True, "gate_vector": True},
}


@pytest.mark.parametrize("fmt_name", list(CUSTOM_FORMATS))
def test_custom_formats_match_oracle(fmt_name, monkeypatch):
    """Formats outside the four compiled-in ones run the kernel whose block
    widths are read at run time; same bar as the named formats."""
    monkeypatch.setitem(W.FORMATS, fmt_name, CUSTOM_FORMATS[fmt_name])
    base = W.WORKLOADS[3] if CUSTOM_FORMATS[fmt_name]["gate_vector"] else W.WORKLOADS[2]
    w = W.Workload(base.index, fmt_name, fmt_name, 7, 11, 2, base.gate_mu, base.gate_sigma, base.seed + 99)
    S = W.initial_state(w)
    fmt, perm, pages = oracle_quantize(w, S.numpy())
    qs = make_state(w)
    qs.calibrate_and_quantize(S.cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(qs.perm().cpu().numpy(), perm)
    assert np.array_equal(download(qs), pages)
    seed = W.sr_seed(w)
    for step in range(w.steps):
        x, xd = step_inputs_gpu(w, step)
        o = qs.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], seed=seed, step=step)
        expect, o_ref = oracle_step(fmt, w, w.batch, w.heads, pages, perm, x, seed, step)
        assert np.array_equal(o.cpu().numpy().reshape(w.pages, 128), o_ref), step
        res = compare_pages(fmt, download(qs), expect, perm, (pages, x, seed, step, w.heads))
        assert res["pages_equal"] == res["pages"], (step, res)
        pages = expect


def test_steps_captured_in_a_cuda_graph_match_eager_steps():
    """Four decode steps captured into one CUDA graph (programmatic launches
    become graph edges) and replayed give the pages and o of eager steps."""
    w = _small("stepquant6", batch=6, heads=7, steps=4)
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    qa, qb = make_state(w), make_state(w)
    upload(qa, perm, pages)
    upload(qb, perm, pages)
    xs = [{k: v.cuda() for k, v in W.step_inputs(w, t).items()} for t in range(4)]
    o_eager = [qa.step(x["q"], x["k"], x["v"], x["alpha"], x["beta"], seed=3, step=t) for t, x in enumerate(xs)]
    torch.cuda.synchronize()
    o_graph = [torch.empty_like(o_eager[0]) for _ in range(4)]
    stream = torch.cuda.Stream()
    B.stq_decode_step(qb.state, xs[0]["q"], xs[0]["k"], xs[0]["v"], xs[0]["alpha"], xs[0]["beta"],
                      torch.empty_like(o_eager[0]), 0, 0, stream)   # first launch outside the capture
    torch.cuda.synchronize()
    upload(qb, perm, pages)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for t, x in enumerate(xs):
            B.stq_decode_step(qb.state, x["q"], x["k"], x["v"], x["alpha"], x["beta"], o_graph[t], 3, t,
                              torch.cuda.current_stream())
    upload(qb, perm, pages)          # the capture ran nothing: start the replay from the same pages
    g.replay()
    torch.cuda.synchronize()
    for t in range(4):
        assert torch.equal(o_graph[t], o_eager[t]), t
    assert torch.equal(qb.pages(), qa.pages())


@pytest.mark.parametrize("n", [1, 2, 5])
def test_pipelined_host_steps_equal_device_steps(n):
    """stq_decode_steps_host (copies overlapped with the steps on side
    streams) gives the o and pages of the same steps run on the device."""
    w = _small("stepquant4_kda", batch=8, heads=6, steps=5)
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    qa, qb = make_state(w), make_state(w)
    upload(qa, perm, pages)
    upload(qb, perm, pages)
    xs = [W.step_inputs(w, t) for t in range(n)]
    o_dev = []
    for t, x in enumerate(xs):
        xd = {k: v.cuda() for k, v in x.items()}
        o_dev.append(qa.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], seed=4, step=10 + t).cpu())
    host = {k: torch.stack([x[k] for x in xs]).contiguous().pin_memory() for k in xs[0]}
    ho = torch.empty(n, 8, 6, 128).pin_memory()
    io_bytes = 2 * B.stq_decode_io_bytes(qb.state)
    io_raw = torch.empty(io_bytes + 256, dtype=torch.uint8, device="cuda")
    off = (-io_raw.data_ptr()) % 256
    B.stq_decode_steps_host(qb.state, host["q"], host["k"], host["v"], host["alpha"], host["beta"], ho,
                            io_raw[off:off + io_bytes], seed=4, step=10)
    torch.cuda.synchronize()
    assert B.stq_device_status(qb.state) == B.STQ_OK
    for t in range(n):
        assert torch.equal(ho[t], o_dev[t]), t
    assert torch.equal(qa.pages(), qb.pages())


def test_pipelined_host_calls_back_to_back():
    """Two stq_decode_steps_host calls of three steps each on one staging
    buffer, with no host synchronization between them (the second call's
    first copies may only start once the first call's steps no longer need
    the slots): the o and pages of six device steps."""
    w = _small("damp", batch=8, heads=6, steps=6)
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    qa, qb = make_state(w), make_state(w)
    upload(qa, perm, pages)
    upload(qb, perm, pages)
    xs = [W.step_inputs(w, t) for t in range(6)]
    o_dev = []
    for t, x in enumerate(xs):
        xd = {k: v.cuda() for k, v in x.items()}
        o_dev.append(qa.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], seed=9, step=t).cpu())
    io_bytes = 2 * B.stq_decode_io_bytes(qb.state)
    io_raw = torch.empty(io_bytes + 256, dtype=torch.uint8, device="cuda")
    off = (-io_raw.data_ptr()) % 256
    io = io_raw[off:off + io_bytes]
    hos = []
    for c in range(2):
        part = xs[3 * c:3 * c + 3]
        host = {k: torch.stack([x[k] for x in part]).contiguous().pin_memory() for k in part[0]}
        ho = torch.full((3, 8, 6, 128), float("nan")).pin_memory()
        B.stq_decode_steps_host(qb.state, host["q"], host["k"], host["v"], host["alpha"], host["beta"], ho, io,
                                seed=9, step=3 * c)
        hos.append((host, ho))      # the host buffers stay alive until the stream is done
    torch.cuda.synchronize()
    assert B.stq_device_status(qb.state) == B.STQ_OK
    for t in range(6):
        assert torch.equal(hos[t // 3][1][t % 3], o_dev[t]), t
    assert torch.equal(qa.pages(), qb.pages())
