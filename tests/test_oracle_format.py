"""Pins of the oracle's packed page layout.

The byte layout is this project's own convention (the pages give none), so it
is pinned by properties any correct packing must have: the size closed form,
an exact bijection between (element, code bit) pairs and code-region bits,
locality (each 16-row block in its own byte range, each 16-byte chunk serving
one column quad), and lossless round trips.  The page sizes are also checked
against the memory arithmetic printed on the pages (tests/golden).
"""
import os

import numpy as np
import pytest

import oracle as O
from linear_attention_recurrent_delta_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fmt(name):
    return O.format_from_spec(W.FORMATS[name])


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split("=", 1)
                vals[k.strip()] = float(v)
    return vals


@pytest.mark.parametrize("name,expect", [("stepquant6", 13312), ("int8row", 16896),
                                         ("stepquant4_kda", 9216), ("damp", 18880)])
def test_page_bytes_closed_form(name, expect):
    spec = W.FORMATS[name]
    codes = sum(rows * 128 * (16 if kind == "fp16" else bits) // 8 for rows, kind, bits in spec["groups"])
    scales = 4 * sum(rows for rows, kind, _ in spec["groups"] if kind == "int")
    scales += 4 * 128 * int(spec["col_scales"])
    assert codes + scales == expect == O.page_bytes(_fmt(name))
    assert expect % 16 == 0


def test_state_memory_matches_the_pages_arithmetic():
    g = _read_golden("pages_memory.txt")
    # 144 MiB FP32 per request = heads x 128 x 128 x 4 bytes
    assert g["heads_per_request"] * 128 * 128 * 4 == g["fp32_mib_per_request"] * 2**20
    # the pages' own ratio, 144 / 28.609 = 5.03x
    assert round(g["fp32_mib_per_request"] / g["packed_mib_per_request"], 2) == g["compression"]
    # DAMP's storage reduction is effective bits over 32: 1 - 9.9/32 = 69.1 %
    assert round(100 * (1 - g["damp_effective_bits"] / 32), 1) == g["damp_storage_reduction_pct"]
    # the library's formats: bits per element including fp32 scales
    for name, bits in (("stepquant6", 6.5), ("int8row", 8.25), ("stepquant4_kda", 4.5), ("damp", 9.21875)):
        assert O.page_bytes(_fmt(name)) * 8 / (128 * 128) == bits


def _uniform_format(kind, bits):
    return O.make_format([(128, kind, bits)], col_scales=True)


def _position_map(fmt, bits):
    """Map every code-region bit to the (element, code bit) it stores, by
    packing 14 pages whose codes spell the element index in binary."""
    n_el = 128 * 128
    n_code_bytes = O.page_bytes(fmt) - 4 * 128 * (O.row_kind(fmt, 0) == 0) - 4 * 128
    ident = np.arange(n_el)
    result = {}
    for t in range(bits):
        acc = np.zeros(n_code_bytes * 8, np.int64)
        present = np.zeros(n_code_bytes * 8, bool)
        for i in range(14):
            sel = (ident >> i) & 1
            page = O.Page(fmt)
            if O.row_kind(fmt, 0) == 0:
                bias = 1 << (bits - 1)
                page.code[:] = (sel.reshape(128, 128) << t) - bias
            else:
                page.code[:] = sel.reshape(128, 128) << t
            raw = O.pack_page(fmt, page)[:n_code_bytes]
            on = np.unpackbits(raw, bitorder="little").astype(bool)
            acc[on] |= 1 << i
            present |= on
        # element 0 never sets a bit; find its position by packing it alone
        page = O.Page(fmt)
        if O.row_kind(fmt, 0) == 0:
            page.code[:] = -(1 << (bits - 1))
            page.code[0, 0] += 1 << t
        else:
            page.code[0, 0] = 1 << t
        on0 = np.unpackbits(O.pack_page(fmt, page)[:n_code_bytes], bitorder="little").astype(bool)
        assert on0.sum() == 1
        present |= on0
        result[t] = (acc, present, on0)
    return result, n_code_bytes


@pytest.mark.parametrize("kind,bits", [("int", 2), ("int", 3), ("int", 4), ("int", 5), ("int", 6),
                                       ("int", 7), ("int", 8), ("fp16", 16)])
def test_pack_is_a_bijection_onto_the_code_region(kind, bits):
    fmt = _uniform_format(kind, bits)
    pm, nbytes = _position_map(fmt, bits)
    assert nbytes == 128 * 128 * bits // 8
    owner = np.full(nbytes * 8, -1, np.int64)
    for t, (acc, present, on0) in pm.items():
        where = np.flatnonzero(present)
        ids = acc[where]
        ids[on0[where]] = 0
        # every element's bit t lands on exactly one page bit, all distinct
        assert np.array_equal(np.sort(ids), np.arange(128 * 128))
        assert np.all(owner[where] == -1)
        owner[where] = ids * 16 + t
    assert np.all(owner >= 0)   # onto: no code-region bit is left unused
    # locality: stored row s lives in block s // 16, a contiguous byte range
    pos = np.flatnonzero(owner >= 0)
    el = owner[pos] // 16
    rows, cols = el // 128, el % 128
    block_bytes = nbytes // 8
    assert np.array_equal(pos // 8 // block_bytes, rows // 16)
    # each 16-byte chunk (8 bytes in a 1-bit plane) serves one column quad;
    # a block holds the planes of the binary decomposition of the width
    widths = [16] if bits == 16 else ([8] if bits == 8 else [w for w in (4, 2, 1) if bits & w])
    in_block = pos // 8 % block_bytes
    plane_start = np.cumsum([0] + [256 * w for w in widths])
    plane = np.searchsorted(plane_start, in_block, side="right") - 1
    chunk = np.where(np.asarray(widths)[plane] == 1, 8, 16)
    chunk_id = (pos // 8 // block_bytes) * 10**6 + plane * 10**4 + (in_block - plane_start[plane]) // chunk
    for cid in np.unique(chunk_id):
        assert len(np.unique(cols[chunk_id == cid] // 4)) == 1


@pytest.mark.parametrize("name", list(W.FORMATS))
def test_pack_unpack_round_trip_random_codes(name):
    fmt = _fmt(name)
    rng = np.random.default_rng(7)
    page = O.Page(fmt)
    for s in range(128):
        qm = O.row_qmax(fmt, s)
        if qm:
            page.code[s] = rng.integers(-qm, qm + 1, 128)
            page.r[s] = np.float32(rng.random() + 0.5)
        else:
            page.code[s] = rng.integers(0, 1 << 16, 128)
    if fmt.col_scales:
        page.c[:] = rng.random(128).astype(np.float32) + 1
    raw = O.pack_page(fmt, page)
    back = O.unpack_page(fmt, raw)
    np.testing.assert_array_equal(back.code, page.code)
    np.testing.assert_array_equal(back.r, page.r)
    np.testing.assert_array_equal(back.c, page.c)
    np.testing.assert_array_equal(O.pack_page(fmt, back), raw)


def test_scale_regions_follow_the_codes():
    fmt = _fmt("stepquant6")
    page = O.Page(fmt)
    page.code[:] = 0
    page.r[:] = np.arange(128, dtype=np.float32) + 1
    page.c[:] = -(np.arange(128, dtype=np.float32) + 1)
    raw = O.pack_page(fmt, page)
    tail = raw[12288:].view(np.float32)
    np.testing.assert_array_equal(tail[:128], page.r)
    np.testing.assert_array_equal(tail[128:], page.c)
    # zero codes are stored biased: the code region holds no zero bytes in INT8 rows
    assert np.all(raw[:4096] == 0x80)
