"""Host-side checks of the C ABI (no GPU needed, no compute call made).

The library loads without a device; every function include/stq.h declares is
exported; the documented host-side argument checks return their status codes
before anything touches CUDA (the pointers passed here are never
dereferenced); page sizes agree with the oracle's, an independent
implementation of the same layout.
"""
import ctypes
import os
import re

import pytest

import oracle as O
from linear_attention_recurrent_delta_b200 import binding as B
from linear_attention_recurrent_delta_b200 import build as build_mod
from linear_attention_recurrent_delta_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.lib()


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(stq_[a-z_0-9]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 16
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert B.stq_version() == 100
    for st in range(7):
        assert B.stq_status_string(st) not in ("", "unknown status")


@pytest.mark.parametrize("name", list(W.FORMATS))
def test_page_bytes_agree_with_the_oracle(lib, name):
    fmt = B.format_from_spec(W.FORMATS[name])
    assert B.stq_page_bytes(fmt) == O.page_bytes(O.format_from_spec(W.FORMATS[name]))


def test_format_validation(lib):
    good = B.make_format([(32, "int", 8), (64, "int", 6), (32, "int", 4)], col_scales=True)
    assert B.stq_page_bytes(good) == 13312
    assert B.stq_page_bytes(B.make_format([(120, "int", 8), (8, "int", 4)])) == 0     # not a multiple of 16
    assert B.stq_page_bytes(B.make_format([(128, "int", 9)])) == 0                    # width
    assert B.stq_page_bytes(B.make_format([(128, "int", 1)])) == 0
    assert B.stq_page_bytes(B.make_format([(112, "int", 8)])) == 0                    # rows do not sum to 128
    assert B.stq_page_bytes(B.make_format([(128, "int", 8)], d_k=64, d_v=64)) == 0    # d != 128
    assert B.stq_page_bytes(B.make_format([(128, "fp16", 0)])) == 128 * 128 * 2
    for bits in range(2, 9):
        assert B.stq_page_bytes(B.make_format([(128, "int", bits)])) == 128 * 128 * bits // 8 + 512
    assert B.stq_state_bytes(good, 0, 4) == 0
    assert B.stq_state_bytes(good, 3, 5) == 256 + 768 + 15 * 13312


FAKE = 1 << 40   # a 256-aligned address that is never dereferenced


def _alloc(lib, fmt, batch, heads, addr=FAKE, nbytes=None):
    h = ctypes.c_void_p()
    n = B.stq_state_bytes(fmt, batch, heads) if nbytes is None else nbytes
    st = lib.stq_state_alloc(ctypes.byref(fmt), batch, heads, ctypes.c_void_p(addr), n, ctypes.byref(h))
    return st, h


def test_state_alloc_checks(lib):
    fmt = B.format_from_spec(W.FORMATS["stepquant6"])
    assert _alloc(lib, fmt, 2, 3)[0] == B.STQ_OK
    assert _alloc(lib, fmt, 0, 3)[0] == B.STQ_ERR_INVALID_ARG
    assert _alloc(lib, fmt, 2, 3, addr=0)[0] == B.STQ_ERR_INVALID_ARG
    assert _alloc(lib, fmt, 2, 3, addr=FAKE + 16)[0] == B.STQ_ERR_MISALIGNED
    assert _alloc(lib, fmt, 2, 3, nbytes=B.stq_state_bytes(fmt, 2, 3) - 1)[0] == B.STQ_ERR_BUFFER_TOO_SMALL
    bad = B.make_format([(128, "int", 9)])
    assert _alloc(lib, bad, 2, 3, nbytes=1 << 20)[0] == B.STQ_ERR_UNSUPPORTED
    st, h = _alloc(lib, fmt, 2, 3)
    vals = [ctypes.c_size_t() for _ in range(4)]
    assert lib.stq_state_layout(h, *[ctypes.byref(v) for v in vals]) == B.STQ_OK
    page, perm, pages, status = (v.value for v in vals)
    assert (page, perm, pages, status) == (13312, 256, 256 + 512, 0)
    assert lib.stq_calibrate_workspace_bytes(h) == 1 * 3 * 128 * 8
    assert lib.stq_decode_io_bytes(h) % 256 == 0
    lib.stq_state_free(h)


def test_decode_step_argument_checks_return_before_cuda(lib):
    fmt = B.format_from_spec(W.FORMATS["stepquant6"])
    st, h = _alloc(lib, fmt, 2, 3)
    assert st == B.STQ_OK
    n = 2 * 3
    vec = n * 128 * 4
    base = 1 << 41
    q, k, v, a, b, o = (base + i * (1 << 24) for i in range(6))
    P = ctypes.c_void_p

    def call(q=q, k=k, v=v, a=a, b=b, o=o, state=h):
        return lib.stq_decode_step(state, P(q), P(k), P(v), P(a), P(b), P(o), 0, 0, None)

    assert call(state=None) == B.STQ_ERR_INVALID_ARG
    assert call(q=0) == B.STQ_ERR_INVALID_ARG
    assert call(o=0) == B.STQ_ERR_INVALID_ARG
    assert call(q=q + 4) == B.STQ_ERR_MISALIGNED
    assert call(o=o + 8) == B.STQ_ERR_MISALIGNED
    assert call(b=b + 2) == B.STQ_ERR_MISALIGNED
    assert call(o=q + vec // 2) == B.STQ_ERR_INVALID_ARG        # output overlaps an input
    assert call(v=FAKE + 1024) == B.STQ_ERR_INVALID_ARG          # input overlaps the state
    assert call(o=FAKE + 512) == B.STQ_ERR_INVALID_ARG           # output overlaps the state
    lib.stq_state_free(h)
    kda = B.format_from_spec(W.FORMATS["stepquant4_kda"])
    st, h = _alloc(lib, kda, 2, 3)
    assert call(a=a + 4, state=h) == B.STQ_ERR_MISALIGNED       # a vector gate needs 16-byte alignment
    lib.stq_state_free(h)


def test_other_entry_points_check_arguments(lib):
    fmt = B.format_from_spec(W.FORMATS["int8row"])
    st, h = _alloc(lib, fmt, 2, 3)
    P = ctypes.c_void_p
    S = 1 << 42
    assert lib.stq_quantize_state(h, None, None) == B.STQ_ERR_INVALID_ARG
    assert lib.stq_quantize_state(h, P(S + 4), None) == B.STQ_ERR_MISALIGNED
    assert lib.stq_quantize_state(h, P(FAKE), None) == B.STQ_ERR_INVALID_ARG   # overlaps the state
    assert lib.stq_dequantize_state(h, P(S + 8), None) == B.STQ_ERR_MISALIGNED
    ws = 1 << 43
    assert lib.stq_calibrate(h, P(S), None, P(ws), 8, None) == B.STQ_ERR_BUFFER_TOO_SMALL
    assert lib.stq_calibrate(h, P(S), None, P(ws + 4), 1 << 20, None) == B.STQ_ERR_MISALIGNED
    assert lib.stq_calibrate(h, P(S), None, None, 1 << 20, None) == B.STQ_ERR_INVALID_ARG
    io = 1 << 44
    hp = P(1 << 45)
    assert lib.stq_decode_step_host(h, hp, hp, hp, hp, hp, hp, P(io), 16, 0, 0, None) == B.STQ_ERR_BUFFER_TOO_SMALL
    assert lib.stq_decode_step_host(h, hp, hp, hp, hp, hp, hp, P(io + 16), 1 << 30, 0, 0, None) == B.STQ_ERR_MISALIGNED
    assert lib.stq_set_wait_limit(None, 0, 0) == B.STQ_ERR_INVALID_ARG
    assert lib.stq_device_status(None, None, 0) == B.STQ_ERR_INVALID_ARG
    lib.stq_state_free(h)


def test_slot_step_and_request_pages_check_arguments(lib):
    fmt = B.format_from_spec(W.FORMATS["int8row"])
    st, h = _alloc(lib, fmt, 4, 3)
    assert st == B.STQ_OK
    P = ctypes.c_void_p
    base = 1 << 41
    q, k, v, a, b, o = (P(base + i * (1 << 24)) for i in range(6))
    table = 1 << 46

    def call(sl=table, n=2):
        return lib.stq_decode_step_slots(h, P(sl) if sl else None, n, q, k, v, a, b, o, 0, 0, None)

    assert call(sl=0) == B.STQ_ERR_INVALID_ARG
    assert call(n=0) == B.STQ_ERR_INVALID_ARG
    assert call(n=5) == B.STQ_ERR_INVALID_ARG          # more rows than the state has requests
    assert call(sl=table + 2) == B.STQ_ERR_MISALIGNED
    assert call(sl=FAKE + 256) == B.STQ_ERR_INVALID_ARG  # the table overlaps the state
    off, nb = ctypes.c_size_t(), ctypes.c_size_t()
    for bad in (-1, 4):
        assert lib.stq_request_pages(h, bad, ctypes.byref(off), ctypes.byref(nb)) == B.STQ_ERR_INVALID_ARG
    assert lib.stq_request_pages(None, 0, None, None) == B.STQ_ERR_INVALID_ARG
    assert lib.stq_request_pages(h, 2, ctypes.byref(off), ctypes.byref(nb)) == B.STQ_OK
    pb, pages_off = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.stq_state_layout(h, ctypes.byref(pb), None, ctypes.byref(pages_off), None) == B.STQ_OK
    assert off.value == pages_off.value + 2 * 3 * pb.value
    assert nb.value == 3 * pb.value
    lib.stq_state_free(h)


def test_window_step_checks_arguments(lib):
    fmt = B.format_from_spec(W.FORMATS["stepquant6"])
    st, h = _alloc(lib, fmt, 2, 3)
    assert st == B.STQ_OK
    P = ctypes.c_void_p
    base = 1 << 41
    q, k, v, a, b, o = (P(base + i * (1 << 24)) for i in range(6))
    for bad in (0, B.STQ_WINDOW_MAX + 1, -3):
        assert lib.stq_window_buffer_bytes(h, bad) == 0
    assert lib.stq_window_buffer_bytes(None, 4) == 0
    assert lib.stq_window_buffer_bytes(h, 4) == 2 * 3 * 512 * 9
    assert lib.stq_window_buffer_bytes(h, B.STQ_WINDOW_MAX) == 2 * 3 * 512 * (1 + 2 * B.STQ_WINDOW_MAX)
    buf = 1 << 46
    need = lib.stq_window_buffer_bytes(h, 4)

    def call(window=4, t=0, commit=0, buf=buf, nbytes=need, q=q, o=o):
        return lib.stq_window_step(h, P(buf) if buf else None, nbytes, window, t, commit, q, k, v, a, b, o, 0, 0,
                                   None)

    assert call(buf=0) == B.STQ_ERR_INVALID_ARG
    assert call(window=0) == B.STQ_ERR_INVALID_ARG
    assert call(window=B.STQ_WINDOW_MAX + 1) == B.STQ_ERR_INVALID_ARG
    assert call(t=-1) == B.STQ_ERR_INVALID_ARG
    assert call(t=4) == B.STQ_ERR_INVALID_ARG
    assert call(t=3, commit=0) == B.STQ_ERR_INVALID_ARG      # a window's last step must commit
    assert call(q=P(base + 4)) == B.STQ_ERR_MISALIGNED
    assert call(buf=buf + 16) == B.STQ_ERR_MISALIGNED
    assert call(nbytes=need - 1) == B.STQ_ERR_BUFFER_TOO_SMALL
    assert call(buf=FAKE) == B.STQ_ERR_INVALID_ARG           # the buffer overlaps the state
    assert call(buf=base) == B.STQ_ERR_INVALID_ARG           # the buffer overlaps q
    assert lib.stq_window_step(None, P(buf), need, 4, 0, 0, q, k, v, a, b, o, 0, 0, None) == B.STQ_ERR_INVALID_ARG
    lib.stq_state_free(h)


@pytest.mark.parametrize("entry", ["stq_prefill", "stq_prefill_chunked"])
def test_prefill_checks_arguments(lib, entry):
    fmt = B.format_from_spec(W.FORMATS["stepquant4_kda"])
    st, h = _alloc(lib, fmt, 2, 3)
    assert st == B.STQ_OK
    P = ctypes.c_void_p
    base = 1 << 41
    q, k, v, a, b, o = (base + i * (1 << 26) for i in range(6))
    S = 1 << 45
    fn = getattr(lib, entry)

    def call(L=4, q=q, a=a, o=o, S_out=None, state=h):
        return fn(state, L, P(q) if q else None, P(k), P(v), P(a), P(b), P(o),
                  P(S_out) if S_out else None, 0, 0, None)

    assert call(state=None) == B.STQ_ERR_INVALID_ARG
    assert call(q=0) == B.STQ_ERR_INVALID_ARG
    assert call(L=0) == B.STQ_ERR_INVALID_ARG
    assert call(L=2**30) == B.STQ_ERR_INVALID_ARG                # L * pages must stay below 2^31
    assert call(q=q + 4) == B.STQ_ERR_MISALIGNED
    assert call(a=a + 4) == B.STQ_ERR_MISALIGNED                  # a vector gate needs 16-byte alignment
    assert call(S_out=S + 8) == B.STQ_ERR_MISALIGNED
    assert call(o=q + 256) == B.STQ_ERR_INVALID_ARG               # output overlaps an input
    assert call(o=FAKE + 512) == B.STQ_ERR_INVALID_ARG            # output overlaps the state
    assert call(S_out=o) == B.STQ_ERR_INVALID_ARG                 # the state output overlaps o
    lib.stq_state_free(h)
    # scalar gates: alpha needs 4-byte alignment
    st, h = _alloc(lib, B.format_from_spec(W.FORMATS["int8row"]), 2, 3)
    assert st == B.STQ_OK
    assert call(a=a + 2, state=h) == B.STQ_ERR_MISALIGNED
    assert call(L=-1, state=h) == B.STQ_ERR_INVALID_ARG
    lib.stq_state_free(h)


def test_lifetime_weights_checks_arguments(lib):
    fmt = B.format_from_spec(W.FORMATS["stepquant4_kda"])
    st, h = _alloc(lib, fmt, 2, 3)
    P = ctypes.c_void_p
    a, w = 1 << 41, 1 << 42
    assert lib.stq_lifetime_weights(None, P(a), 4, P(w), None) == B.STQ_ERR_INVALID_ARG
    assert lib.stq_lifetime_weights(h, None, 4, P(w), None) == B.STQ_ERR_INVALID_ARG
    assert lib.stq_lifetime_weights(h, P(a), 0, P(w), None) == B.STQ_ERR_INVALID_ARG
    assert lib.stq_lifetime_weights(h, P(a + 4), 4, P(w), None) == B.STQ_ERR_MISALIGNED   # vector gates: 16 bytes
    assert lib.stq_lifetime_weights(h, P(a), 4, P(w + 8), None) == B.STQ_ERR_MISALIGNED
    assert lib.stq_lifetime_weights(h, P(a), 4, P(a + 256), None) == B.STQ_ERR_INVALID_ARG   # output overlaps the gates
    assert lib.stq_lifetime_weights(h, P(FAKE), 4, P(w), None) == B.STQ_ERR_INVALID_ARG     # gates overlap the state
    lib.stq_state_free(h)


def test_pipelined_host_steps_check_arguments(lib):
    fmt = B.format_from_spec(W.FORMATS["int8row"])
    st, h = _alloc(lib, fmt, 2, 3)
    P = ctypes.c_void_p
    hp = P(1 << 45)
    io = 1 << 44
    need = lib.stq_decode_io_bytes(h)

    def call(n=3, io=io, nbytes=2 * need):
        return lib.stq_decode_steps_host(h, n, hp, hp, hp, hp, hp, hp, P(io), nbytes, 0, 0, None)

    assert call(n=0) == B.STQ_ERR_INVALID_ARG
    assert call(nbytes=2 * need - 1) == B.STQ_ERR_BUFFER_TOO_SMALL   # two staging slots
    assert call(io=io + 16) == B.STQ_ERR_MISALIGNED
    assert call(io=FAKE) == B.STQ_ERR_INVALID_ARG                    # staging overlaps the state
    lib.stq_state_free(h)
