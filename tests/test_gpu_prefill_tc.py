"""GPU parity of the chunkwise tensor-core prefill (stq_prefill_chunked).

The kernel resolves the prompt 128 tokens at a time with tf32 tensor-core
products on split operands and a triangular solve, so it agrees with the
token recurrence to fp32 rounding, not bit for bit.  The bar, per page:
  * o of every token and the final fp32 state (the optional state output)
    within rel-L2 1e-5 of the oracle's chunk algebra in fp64
    (orc_prefill_chunked_f64, itself pinned against the recurrence), and
    within 1e-5 of the recurrent GPU prefill run on the same inputs;
  * the requantized page is the requantization of the kernel's own final
    state: each row scale is that state's row maximum / qmax (to 2 ulps), each
    INT code the nearest integer to x = T qmax / m (with the stochastic
    offset of the oracle's generator for stochastic formats) except within
    1e-5 of a rounding midpoint, each FP16 row element the binary16 rounding
    of T except at a near-tie.
Prompts of 1, 37, 128, 130 and 300 tokens (one chunk, a ragged chunk, two
and three chunks); the GDN formats and KDA's gate vectors; zero and
vanishing gates; more pages than SMs for the persistent grid; the
bounded-wait hook.
"""
import numpy as np
import pytest
import torch

import oracle as O
from linear_attention_recurrent_delta_b200 import binding as B
from linear_attention_recurrent_delta_b200 import workloads as W

from parity_util import download, make_state, oracle_quantize, rel_l2, upload

pytestmark = pytest.mark.gpu

GDN = ["int8row", "stepquant6", "damp"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from linear_attention_recurrent_delta_b200 import build
    build.build()
    B.lib()
    assert torch.cuda.is_available()


def _setup(name, batch, heads):
    w = [x for x in W.WORKLOADS if x.fmt == name and x.index > 0][0].resized(batch=batch, heads=heads, steps=2)
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    qs = make_state(w)
    upload(qs, perm, pages)
    return w, fmt, perm, pages, qs


def _prompt(w, L, first=0):
    xs = [W.step_inputs(w, first + l) for l in range(L)]
    return {k: torch.stack([x[k] for x in xs]).contiguous() for k in xs[0]}


def _check_requant(fmt, page, T, seed, step, b, h):
    """page: the kernel's packed page (unpacked); T: its final state in stored
    order, column-normalised (double).  Returns the number of codes within
    the near-tie band (allowed either way).  With column scales, T is
    recovered as S / c from the fp32 state output S = fl(T c): one fp32
    rounding, |error| <= 2^-24 |T|, so the band widens by that error in the
    rounding's own units (x's for INT rows, binary16 ulps for FP16 rows)."""
    rel = 2.0 ** -23 if fmt.col_scales else 0.0   # the recovery's error, with margin (x2)
    ties = 0
    for s in range(128):
        kind = O.row_kind(fmt, s)
        t = T[s]
        if kind == 1:
            h16 = O.f16_to_f32(page.code[s].astype(np.uint16)).astype(np.float64)
            ax = np.abs(t)
            sp = np.where(ax < 2.0 ** -14, 2.0 ** -24, 2.0 ** (np.floor(np.log2(np.maximum(ax, 2.0 ** -14))) - 10))
            err = np.abs(h16 - t) / sp
            band = 1e-5 + rel * ax / sp
            assert np.all(err <= 0.5 + band), (s, err.max())
            ties += int(np.sum(err > 0.5 - band))
            continue
        qmax = O.row_qmax(fmt, s)
        m = np.abs(t).max()
        r = float(page.r[s])
        assert abs(r - m / qmax) <= 2 * np.spacing(np.float32(m / qmax)), (s, r, m / qmax)
        if m == 0:
            assert np.all(page.code[s] == 0)
            continue
        x = t * qmax / m
        band = 1e-5 + 2 * rel * np.abs(x)           # t and the row maximum m each carry the error
        if fmt.stochastic:
            # floor(x + u) lies within 1/2 of x + u - 1/2
            x = x + np.array([O.sr_offset(seed, step, b, h, s, j) for j in range(128)], np.float64) - 0.5
        z = page.code[s].astype(np.float64)
        d = np.abs(z - x)
        assert np.all(d <= 0.5 + band), (s, d.max())
        ties += int(np.sum(d > 0.5 - band))
    return ties


@pytest.mark.parametrize("L", [1, 37, 128, 130, 300])
@pytest.mark.parametrize("name", GDN)
def test_chunked_prefill_matches_the_chunk_algebra(name, L):
    w, fmt, perm, pages, qs = _setup(name, 3, 5)
    _check_chunked(name, w, fmt, perm, pages, qs, _prompt(w, L), L)


@pytest.mark.parametrize("name", ["stepquant6", "damp"])
def test_zero_and_vanishing_gates(name):
    """A gate of zero, and a run of 0.4 gates whose cumulative product leaves
    the float range inside a chunk (0.4^128 ~ 1e-51): the decay between two
    tokens is a product of gates in the kernel too, so o and the state stay
    finite and within the bar of the chunk algebra and of the recurrence."""
    w, fmt, perm, pages, qs = _setup(name, 3, 5)
    L = 300
    x = _prompt(w, L)
    a = x["alpha"].clone()
    a[3, 0] = 0.0                       # request 0: one token forgets everything
    a[10:200, 1] = 0.4                  # request 1: the cumulative decay underflows
    a[130:260:7, 2] = 0.0               # request 2: zero gates in the second chunk
    x["alpha"] = a.contiguous()
    _check_chunked(name, w, fmt, perm, pages, qs, x, L)


def _check_chunked(name, w, fmt, perm, pages, qs, x, L):
    xd = {k: v.cuda() for k, v in x.items()}
    o = torch.full((L, w.batch, w.heads, 128), float("nan"), device="cuda")
    S_out = torch.empty(w.batch, w.heads, 128, 128, device="cuda")
    seed = W.sr_seed(w)
    B.stq_prefill_chunked(qs.state, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o, S_out, seed, 7)
    assert B.stq_device_status(qs.state) == B.STQ_OK
    got = download(qs)
    o_g, S_g = o.cpu().numpy(), S_out.cpu().numpy()
    # the recurrent GPU prefill on the same inputs
    qr = make_state(w)
    upload(qr, perm, pages)
    o_r = torch.empty_like(o)
    S_r = torch.empty_like(S_out)
    B.stq_prefill(qr.state, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o_r, S_r, seed, 7)
    o_r, S_r = o_r.cpu().numpy(), S_r.cpu().numpy()
    ties, worst_o, worst_s = 0, 0.0, 0.0
    for i in range(w.pages):
        b, h = divmod(i, w.heads)
        page0 = O.unpack_page(fmt, pages[i])
        o64, S64 = O.prefill_chunked_f64(fmt, page0, perm[h], x["q"][:, b, h].numpy(), x["k"][:, b, h].numpy(),
                                         x["v"][:, b, h].numpy(), x["alpha"][:, b, h].numpy(),
                                         x["beta"][:, b, h].numpy(), 128)
        worst_o = max(worst_o, rel_l2(o_g[:, b, h], o64))
        worst_s = max(worst_s, rel_l2(S_g[b, h], S64))
        assert rel_l2(o_g[:, b, h], o64) <= 1e-5, ("o", i, rel_l2(o_g[:, b, h], o64))
        assert rel_l2(S_g[b, h], S64) <= 1e-5, ("state", i, rel_l2(S_g[b, h], S64))
        assert rel_l2(o_g[:, b, h], o_r[:, b, h]) <= 1e-5
        assert rel_l2(S_g[b, h], S_r[b, h]) <= 1e-5
        pg = O.unpack_page(fmt, got[i])
        c = page0.c.astype(np.float64) if fmt.col_scales else np.ones(128)
        T = S_g[b, h].astype(np.float64)[perm[h]] / c           # stored order, column-normalised
        assert np.array_equal(pg.c.view(np.uint32), page0.c.view(np.uint32))
        ties += _check_requant(fmt, pg, T, seed, 7, b, h)
    print("\n%s, L = %d: max o rel-L2 %.2e, max state rel-L2 %.2e, near-tie codes %d"
          % (name, L, worst_o, worst_s, ties))


@pytest.mark.parametrize("name", ["int8row", "stepquant4_kda"])
def test_many_pages_per_cta(name):
    """More pages than SMs: every CTA takes several pages in turn (gate
    vectors: some of them token by token, zero gates on every fifth page)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    w, fmt, perm, pages, qs = _setup(name, (sms * 2) // 4 + 3, 4)
    L = 20
    x = _prompt(w, L)
    if fmt.gate_vector:
        a = x["alpha"].clone()
        a.view(L, -1, 128)[4, ::5, :] = 0.0
        x["alpha"] = a.contiguous()
    xd = {k: v.cuda() for k, v in x.items()}
    o = torch.empty(L, w.batch, w.heads, 128, device="cuda")
    B.stq_prefill_chunked(qs.state, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o, None, 0, 3)
    assert B.stq_device_status(qs.state) == B.STQ_OK
    o_g = o.cpu().numpy()
    for i in (0, w.pages // 2, w.pages - 1):
        b, h = divmod(i, w.heads)
        o64, _ = O.prefill_chunked_f64(fmt, O.unpack_page(fmt, pages[i]), perm[h], x["q"][:, b, h].numpy(),
                                       x["k"][:, b, h].numpy(), x["v"][:, b, h].numpy(),
                                       x["alpha"][:, b, h].numpy(), x["beta"][:, b, h].numpy(), 128)
        assert rel_l2(o_g[:, b, h], o64) <= 1e-5


@pytest.mark.parametrize("L", [1, 37, 128, 130, 300])
def test_vector_gates_match_the_chunk_algebra(L):
    """KDA gates (a vector over key channels): the decays Gam of every channel
    folded into the operands (K Gam, Q Gam, K / Gam), the same bars."""
    w, fmt, perm, pages, qs = _setup("stepquant4_kda", 3, 5)
    _check_chunked("stepquant4_kda", w, fmt, perm, pages, qs, _prompt(w, L), L)


def test_vector_gates_zero_and_vanishing():
    """Chunks whose per-channel decays leave the range run token by token on
    the CUDA cores: a zero gate on some channels, and a run of 0.2 gates on
    others (0.2^128 ~ 1e-90), next to chunks of the matrix form."""
    w, fmt, perm, pages, qs = _setup("stepquant4_kda", 3, 5)
    L = 300
    x = _prompt(w, L)
    a = x["alpha"].clone()
    a[3, 0, :, ::5] = 0.0               # request 0: some channels forget at token 3
    a[10:200, 1, :, 7] = 0.2            # request 1: one channel's decay underflows
    a[130:260:7, 2] = 0.0               # request 2: every channel forgets, second chunk
    x["alpha"] = a.contiguous()
    _check_chunked("stepquant4_kda", w, fmt, perm, pages, qs, x, L)


@pytest.mark.parametrize("name", ["stepquant6", "stepquant4_kda"])
def test_bounded_wait_times_out_and_writes_nothing(name):
    w, fmt, perm, pages, qs = _setup(name, 4, 3)
    L = 40
    x = _prompt(w, L)
    xd = {k: v.cuda() for k, v in x.items()}
    o = torch.full((L, 4, 3, 128), 7.0, device="cuda")
    B.stq_set_wait_limit(qs.state, 20_000_000, stall_first_wait=True)
    B.stq_prefill_chunked(qs.state, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o, None, 0, 1)
    assert B.stq_device_status(qs.state, clear=True) == B.STQ_ERR_DEVICE_TIMEOUT
    assert np.array_equal(download(qs), pages)
    assert bool((o == 7.0).all())
    B.stq_set_wait_limit(qs.state, 0, stall_first_wait=False)
    B.stq_prefill_chunked(qs.state, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o, None, 0, 1)
    assert B.stq_device_status(qs.state) == B.STQ_OK
    o_g = o.cpu().numpy()
    b, h = 1, 2
    o64, _ = O.prefill_chunked_f64(fmt, O.unpack_page(fmt, pages[b * 3 + h]), perm[h], x["q"][:, b, h].numpy(),
                                   x["k"][:, b, h].numpy(), x["v"][:, b, h].numpy(), x["alpha"][:, b, h].numpy(),
                                   x["beta"][:, b, h].numpy(), 128)
    assert rel_l2(o_g[:, b, h], o64) <= 1e-5


def _tc_sample_positions(n, seed):
    """Pages to check in a full-size launch: every page when there are few,
    else the ends, both sides of each wrap of the one-CTA-per-SM persistent
    grid, and seeded random positions."""
    if n <= 64:
        return list(range(n))
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    pos = {0, 1, n - 2, n - 1}
    for m in (1, 2, n // sms):
        for d in (-1, 0):
            if 0 <= m * sms + d < n:
                pos.add(m * sms + d)
    rng = np.random.default_rng(seed)
    pos.update(int(x) for x in rng.integers(0, n, 10))
    return sorted(pos)


SMALL_BATCH = 4   # CPU-generated requests the sampled pages are drawn from


@pytest.mark.parametrize("name,batch,L", [("damp", 256, 512), ("damp", 1, 1024), ("stepquant4_kda", 1, 1024)])
def test_full_size_chunked_prefill_on_sampled_pages(name, batch, L):
    """The benchmark's launch configurations of stq_prefill_chunked (256
    requests x 32 heads x 512 tokens; one request x 32 heads x 1,024 tokens,
    scalar gates and gate vectors), checked on sampled pages against the
    fp64 chunk algebra.  The state is the GPU's quantization of a
    device-generated fp32 state except at the sampled positions, which hold
    oracle-made pages of a small CPU-generated batch with CPU-generated
    prompts; the bar is the one above (o and final state within rel-L2
    1e-5, the requantized page the requantization of the kernel's state)."""
    w = [x for x in W.WORKLOADS if x.fmt == name and x.index > 0][0].resized(batch=batch)
    H, n = w.heads, w.pages
    fmt = O.format_from_spec(w.format)
    S_small = W.initial_state(w, batch=SMALL_BATCH).numpy()
    perm = O.rank_rows(fmt, S_small)
    pos = _tc_sample_positions(n, w.seed + 5)
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

    xd = {k: torch.stack([W.step_inputs(w, l, device="cuda")[k] for l in range(L)]).contiguous()
          for k in ("q", "k", "v", "alpha", "beta")}
    xc = [W.step_inputs(w, l, batch=SMALL_BATCH) for l in range(L)]
    for k in xd:
        flat = xd[k].view(L, n, -1)
        flat[:, idx] = torch.stack([torch.stack([xc[l][k][b, h].reshape(-1) for b, h in src])
                                    for l in range(L)]).cuda()
    seed = W.sr_seed(w)
    o = torch.full((L, w.batch, H, 128), float("nan"), device="cuda")
    S_out = torch.empty(w.batch, H, 128, 128, device="cuda")
    B.stq_prefill_chunked(qs.state, xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"], o, S_out, seed, 3)
    assert B.stq_device_status(qs.state) == B.STQ_OK
    got_o = o.view(L, n, 128)[:, idx].cpu().numpy()
    got_S = S_out.view(n, 128, 128)[idx].cpu().numpy()
    got_pages = qs.pages()[idx].cpu().numpy()
    del xd, o, S_out
    ties, worst_o, worst_s = 0, 0.0, 0.0
    for i, (p, (b, h)) in enumerate(zip(pos, src)):
        arr = {k: np.stack([xc[l][k][b, h].numpy() for l in range(L)]) for k in ("q", "k", "v", "alpha", "beta")}
        o64, S64 = O.prefill_chunked_f64(fmt, pages[i], perm[h], arr["q"], arr["k"], arr["v"], arr["alpha"],
                                         arr["beta"], 128)
        eo, es = rel_l2(got_o[:, i], o64), rel_l2(got_S[i], S64)
        worst_o, worst_s = max(worst_o, eo), max(worst_s, es)
        assert eo <= 1e-5, ("o", p, eo)
        assert es <= 1e-5, ("state", p, es)
        pg = O.unpack_page(fmt, got_pages[i])
        c = pages[i].c.astype(np.float64) if fmt.col_scales else np.ones(128)
        T = got_S[i].astype(np.float64)[perm[h]] / c
        assert np.array_equal(pg.c.view(np.uint32), pages[i].c.view(np.uint32))
        ties += _check_requant(fmt, pg, T, seed, 3, p // H, p % H)
    print("\n%s, %d x %d pages, L = %d, %d sampled: max o rel-L2 %.2e, max state rel-L2 %.2e, near-tie codes %d"
          % (name, w.batch, H, L, len(pos), worst_o, worst_s, ties))


@pytest.mark.parametrize("gate_vector", [False, True])
@pytest.mark.parametrize("stochastic", [False, True])
def test_runtime_format(gate_vector, stochastic, monkeypatch):
    """A format outside the four compiled-in ones (block widths read at run
    time, an FP16 block between INT blocks), both gate forms, both rounding
    modes: the same bars over a prompt of two chunks and a ragged tail."""
    name = "tc_runtime_%d%d" % (gate_vector, stochastic)
    spec = {"groups": [(32, "int", 7), (16, "fp16", 0), (48, "int", 5), (32, "int", 2)], "col_scales": True,
            "gate_vector": gate_vector, "stochastic": stochastic}
    monkeypatch.setitem(W.FORMATS, name, spec)
    base = [w for w in W.WORKLOADS if w.fmt == ("stepquant4_kda" if gate_vector else "stepquant6") and w.index > 0][0]
    monkeypatch.setattr(W, "WORKLOADS", list(W.WORKLOADS) + [
        W.Workload(base.index, name, name, 3, 5, 2, base.gate_mu, base.gate_sigma, base.seed + 11)])
    w, fmt, perm, pages, qs = _setup(name, 3, 5)
    _check_chunked(name, w, fmt, perm, pages, qs, _prompt(w, 260), 260)
