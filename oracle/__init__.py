"""Python view of the CPU oracle (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and bench.py's CPU legs may
import this package.  It loads ``oracle/libstq_oracle.so`` (built from
``stq_oracle.cpp`` on first use) through ctypes and passes numpy arrays; it
never imports the CUDA library or the product package.

A format is described by plain data, the same description the workload
module uses: ``groups`` is a list of ``(rows, kind, bits)`` with kind one of
``"int"``, ``"fp16"``, ``"fp32"`` (bits ignored for float kinds).
"""
import ctypes
import os
from ctypes import c_int, c_long, c_float, c_uint16, c_uint32, c_uint64, POINTER

import numpy as np

from .build import build as _build

KIND = {"int": 0, "fp16": 1, "fp32": 2}
MAX_GROUPS = 8


class OrcFormat(ctypes.Structure):
    _fields_ = [("d_k", c_int), ("d_v", c_int), ("n_groups", c_int),
                ("group_rows", c_int * MAX_GROUPS), ("group_kind", c_int * MAX_GROUPS),
                ("group_bits", c_int * MAX_GROUPS), ("col_scales", c_int),
                ("stochastic", c_int), ("gate_vector", c_int)]


class _OrcPage(ctypes.Structure):
    _fields_ = [("code", POINTER(ctypes.c_int32)), ("r", POINTER(c_float)),
                ("c", POINTER(c_float))]


_lib = None


def lib():
    global _lib
    if _lib is None:
        # STQ_ORACLE_LIB points the wrapper at another build of the same
        # source (the mutation tests load deliberately broken copies)
        path = os.environ.get("STQ_ORACLE_LIB") or _build()
        _lib = ctypes.CDLL(path)
        L = _lib
        P = ctypes.c_void_p
        L.orc_format_check.argtypes = [P]
        L.orc_row_qmax.argtypes = [P, c_int]
        L.orc_row_kind.argtypes = [P, c_int]
        L.orc_page_bytes.argtypes = [P]
        L.orc_page_bytes.restype = c_long
        L.orc_rank_rows.argtypes = [P, c_int, c_int, P, P, P]
        L.orc_quantize_page.argtypes = [P, P, P, P]
        L.orc_dequantize_page.argtypes = [P, P, P, P]
        L.orc_quantize_page_fit.argtypes = [P, P, P, P, c_int, P, P]
        L.orc_step_f32.argtypes = [P, P, P, P, P, P, P, c_float, P, c_uint64, c_uint32,
                                   c_uint32, c_uint32, P, P]
        L.orc_step_f32_plain.argtypes = L.orc_step_f32.argtypes
        L.orc_step_f64.argtypes = [P, P, P, P, P, P, P, c_float, P, P]
        L.orc_lifetime_weights.argtypes = [P, c_int, c_int, c_int, P, P]
        L.orc_prefill_f32.argtypes = [P, P, P, c_int, P, P, P, P, P, P, c_uint64, c_uint32, c_uint32, c_uint32,
                                      P, P]
        L.orc_window_step_f32.argtypes = [P, P, P, P, P, P, c_int, c_int, P, P, P, P, c_float, P, c_uint64,
                                          c_uint32, c_uint32, c_uint32, P]
        L.orc_window_step_f32_plain.argtypes = L.orc_window_step_f32.argtypes
        L.orc_prefill_f32_plain.argtypes = L.orc_prefill_f32.argtypes
        L.orc_prefill_chunked_f64.argtypes = [P, P, P, c_int, c_int, P, P, P, P, P, P, P]
        L.orc_pack_page.argtypes = [P, P, P]
        L.orc_unpack_page.argtypes = [P, P, P]
        L.orc_decode_step_pages.argtypes = [P, c_int, c_int, P, P, P, P, P, P, P, P,
                                            c_uint64, c_uint32, c_long, c_long]
        L.orc_decode_step_pages_plain.argtypes = L.orc_decode_step_pages.argtypes
        L.orc_f32_to_f16_rn.argtypes = [c_float]
        L.orc_f32_to_f16_rn.restype = c_uint16
        L.orc_f16_to_f32.argtypes = [c_uint16]
        L.orc_f16_to_f32.restype = c_float
        L.orc_div_rz.argtypes = [c_float, c_float]
        L.orc_div_rz.restype = c_float
        L.orc_f32_to_f16_rn_n.argtypes = [P, P, c_long]
        L.orc_f16_to_f32_n.argtypes = [P, P, c_long]
        L.orc_div_rz_n.argtypes = [P, P, P, c_long]
        L.orc_pcg4d.argtypes = [P, P]
        L.orc_sr_offset.argtypes = [c_uint64, c_uint32, c_uint32, c_uint32, c_int, c_int, c_int]
        L.orc_sr_offset.restype = c_float
    return _lib


def _p(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _ok(rc, what):
    if rc != 0:
        raise ValueError("oracle %s failed with %d" % (what, rc))


def make_format(groups, d_k=128, d_v=128, col_scales=False, stochastic=False,
                gate_vector=False):
    f = OrcFormat()
    f.d_k, f.d_v, f.n_groups = d_k, d_v, len(groups)
    for i, (rows, kind, bits) in enumerate(groups):
        f.group_rows[i] = rows
        f.group_kind[i] = KIND[kind]
        f.group_bits[i] = bits if kind == "int" else 0
    f.col_scales, f.stochastic, f.gate_vector = int(col_scales), int(stochastic), int(gate_vector)
    _ok(lib().orc_format_check(ctypes.byref(f)), "format_check")
    return f


def format_from_spec(spec, d_k=128, d_v=128):
    """spec: the plain dict a workload carries (groups, col_scales, stochastic, gate_vector)."""
    return make_format(spec["groups"], d_k, d_v, spec["col_scales"], spec["stochastic"],
                       spec["gate_vector"])


class Page:
    """Unpacked page: code [d_k, d_v] int32 (stored order), r [d_k], c [d_v]."""

    def __init__(self, fmt, code=None, r=None, c=None):
        self.code = np.zeros((fmt.d_k, fmt.d_v), np.int32) if code is None else np.ascontiguousarray(code, np.int32)
        self.r = np.zeros(fmt.d_k, np.float32) if r is None else np.ascontiguousarray(r, np.float32)
        self.c = np.ones(fmt.d_v, np.float32) if c is None else np.ascontiguousarray(c, np.float32)

    def copy(self):
        p = Page.__new__(Page)
        p.code, p.r, p.c = self.code.copy(), self.r.copy(), self.c.copy()
        return p

    def _struct(self):
        return _OrcPage(self.code.ctypes.data_as(POINTER(ctypes.c_int32)),
                        self.r.ctypes.data_as(POINTER(c_float)),
                        self.c.ctypes.data_as(POINTER(c_float)))


def row_qmax(fmt, s):
    return lib().orc_row_qmax(ctypes.byref(fmt), s)


def row_kind(fmt, s):
    return lib().orc_row_kind(ctypes.byref(fmt), s)


def page_bytes(fmt):
    n = lib().orc_page_bytes(ctypes.byref(fmt))
    if n < 0:
        raise ValueError("format has no packed layout")
    return n


def rank_rows(fmt, S, row_weight=None):
    S = np.ascontiguousarray(S, np.float32)
    B, H = S.shape[0], S.shape[1]
    assert S.shape[2:] == (fmt.d_k, fmt.d_v)
    perm = np.zeros((H, fmt.d_k), np.int32)
    rw = None if row_weight is None else np.ascontiguousarray(row_weight, np.float32)
    _ok(lib().orc_rank_rows(ctypes.byref(fmt), B, H, _p(S), _p(rw), _p(perm)), "rank_rows")
    return perm


def lifetime_weights(fmt, alpha):
    """Row weights [H, d_k] from gate samples alpha [n_samples, B, H] or
    [n_samples, B, H, d_k] (gate_vector)."""
    alpha = np.ascontiguousarray(alpha, np.float32)
    n, B, H = alpha.shape[:3]
    w = np.zeros((H, fmt.d_k), np.float32)
    _ok(lib().orc_lifetime_weights(ctypes.byref(fmt), B, H, n, _p(alpha), _p(w)), "lifetime_weights")
    return w


def quantize_page(fmt, S_nat, perm):
    S_nat = np.ascontiguousarray(S_nat, np.float32)
    perm = np.ascontiguousarray(perm, np.int32)
    page = Page(fmt)
    st = page._struct()
    _ok(lib().orc_quantize_page(ctypes.byref(fmt), _p(S_nat), _p(perm), ctypes.byref(st)), "quantize")
    return page


def quantize_page_fit(fmt, S_nat, perm, impact=None, iters=4):
    """Joint fit of the row and column scales (alternating weighted least
    squares from the absmax scales).  Returns (page, objective per round)."""
    S_nat = np.ascontiguousarray(S_nat, np.float32)
    perm = np.ascontiguousarray(perm, np.int32)
    w = None if impact is None else np.ascontiguousarray(impact, np.float32)
    page = Page(fmt)
    st = page._struct()
    err = np.zeros(iters + 1, np.float64)
    _ok(lib().orc_quantize_page_fit(ctypes.byref(fmt), _p(S_nat), _p(perm), _p(w), int(iters), ctypes.byref(st),
                                    _p(err)), "quantize_page_fit")
    return page, err


def dequantize_page(fmt, page, perm):
    perm = np.ascontiguousarray(perm, np.int32)
    out = np.zeros((fmt.d_k, fmt.d_v), np.float32)
    st = page._struct()
    _ok(lib().orc_dequantize_page(ctypes.byref(fmt), ctypes.byref(st), _p(perm), _p(out)), "dequantize")
    return out


def _gate(fmt, alpha):
    a = np.ascontiguousarray(np.atleast_1d(np.asarray(alpha, np.float32)))
    assert a.size == (fmt.d_k if fmt.gate_vector else 1)
    return a


def step_f32(fmt, page, perm, q, k, v, alpha, beta, seed=0, step=0, b=0, h=0,
             want_tp=False, want_margin=False, plain=False):
    """fp32 step; updates ``page`` in place.  Returns (o, Tp, margin).  The
    canonical (kernel) summation order, or with plain=True every column sum
    one fma chain over the key channels in natural order."""
    perm = np.ascontiguousarray(perm, np.int32)
    q, k, v = (np.ascontiguousarray(x, np.float32) for x in (q, k, v))
    a = _gate(fmt, alpha)
    o = np.zeros(fmt.d_v, np.float32)
    tp = np.zeros((fmt.d_k, fmt.d_v), np.float32) if want_tp else None
    mg = np.zeros((fmt.d_k, fmt.d_v), np.float64) if want_margin else None
    st = page._struct()
    fn = lib().orc_step_f32_plain if plain else lib().orc_step_f32
    _ok(fn(ctypes.byref(fmt), ctypes.byref(st), _p(perm), _p(q), _p(k), _p(v),
           _p(a), float(beta), _p(o), int(seed), int(step), int(b), int(h),
           _p(tp), _p(mg)), "step_f32")
    return o, tp, mg


def window_step_f32(fmt, page, perm, P, K, D, t, commit, q, k, v, alpha, beta, seed=0, step=0, b=0, h=0,
                    want_margin=False, plain=False):
    """Per-window decode step t (0-based) on one page; P [d_k], K [W, d_k], D [W, d_v]
    (float32, updated in place; page updated in place when commit).  Returns (o, margin)."""
    perm = np.ascontiguousarray(perm, np.int32)
    q, k, v = (np.ascontiguousarray(x, np.float32) for x in (q, k, v))
    for arr in (P, K, D):
        assert arr.dtype == np.float32 and arr.flags["C_CONTIGUOUS"]
    a = _gate(fmt, alpha)
    o = np.zeros(fmt.d_v, np.float32)
    mg = np.zeros((fmt.d_k, fmt.d_v), np.float64) if (want_margin and commit) else None
    st = page._struct()
    fn = lib().orc_window_step_f32_plain if plain else lib().orc_window_step_f32
    _ok(fn(ctypes.byref(fmt), ctypes.byref(st), _p(perm), _p(P), _p(K), _p(D), int(t),
           int(commit), _p(q), _p(k), _p(v), _p(a), float(beta), _p(o), int(seed),
           int(step), int(b), int(h), _p(mg)), "window_step_f32")
    return o, mg


def prefill_f32(fmt, page, perm, q, k, v, alpha, beta, seed=0, step=0, b=0, h=0, want_tp=False,
                want_margin=False, plain=False):
    """A prompt of L tokens through one page (page requantized in place at
    the end).  q, k, v: [L, 128]; alpha: [L] or [L, 128]; beta: [L].
    Returns (o [L, d_v], T before requantization or None, margin or None)."""
    perm = np.ascontiguousarray(perm, np.int32)
    q, k, v = (np.ascontiguousarray(x, np.float32) for x in (q, k, v))
    L = q.shape[0]
    a = np.ascontiguousarray(np.asarray(alpha, np.float32).reshape(L, -1)[:, :fmt.d_k if fmt.gate_vector else 1])
    bt = np.ascontiguousarray(np.asarray(beta, np.float32).reshape(L))
    o = np.zeros((L, fmt.d_v), np.float32)
    tp = np.zeros((fmt.d_k, fmt.d_v), np.float32) if want_tp else None
    mg = np.zeros((fmt.d_k, fmt.d_v), np.float64) if want_margin else None
    st = page._struct()
    fn = lib().orc_prefill_f32_plain if plain else lib().orc_prefill_f32
    _ok(fn(ctypes.byref(fmt), ctypes.byref(st), _p(perm), int(L), _p(q), _p(k), _p(v), _p(a),
           _p(bt), _p(o), int(seed), int(step), int(b), int(h), _p(tp), _p(mg)), "prefill_f32")
    return o, tp, mg


def prefill_chunked_f64(fmt, page, perm, q, k, v, alpha, beta, chunk):
    """The chunk algebra of a prompt in fp64 from the page (unchanged).
    Returns (o [L, d_v], final state [d_k, d_v] natural order), double."""
    perm = np.ascontiguousarray(perm, np.int32)
    q, k, v = (np.ascontiguousarray(x, np.float32) for x in (q, k, v))
    L = q.shape[0]
    a = np.ascontiguousarray(np.asarray(alpha, np.float32).reshape(L, -1)[:, :fmt.d_k if fmt.gate_vector else 1])
    bt = np.ascontiguousarray(np.asarray(beta, np.float32).reshape(L))
    o = np.zeros((L, fmt.d_v), np.float64)
    sp = np.zeros((fmt.d_k, fmt.d_v), np.float64)
    st = page._struct()
    _ok(lib().orc_prefill_chunked_f64(ctypes.byref(fmt), ctypes.byref(st), _p(perm), int(L), int(chunk), _p(q), _p(k),
                                      _p(v), _p(a), _p(bt), _p(o), _p(sp)), "prefill_chunked_f64")
    return o, sp


def step_f64(fmt, page, perm, q, k, v, alpha, beta):
    """Plain-definition fp64 step (page unchanged).  Returns (o, S') in double."""
    perm = np.ascontiguousarray(perm, np.int32)
    q, k, v = (np.ascontiguousarray(x, np.float32) for x in (q, k, v))
    a = _gate(fmt, alpha)
    o = np.zeros(fmt.d_v, np.float64)
    sp = np.zeros((fmt.d_k, fmt.d_v), np.float64)
    st = page._struct()
    _ok(lib().orc_step_f64(ctypes.byref(fmt), ctypes.byref(st), _p(perm), _p(q), _p(k), _p(v),
                           _p(a), float(beta), _p(o), _p(sp)), "step_f64")
    return o, sp


def pack_page(fmt, page):
    out = np.zeros(page_bytes(fmt), np.uint8)
    st = page._struct()
    _ok(lib().orc_pack_page(ctypes.byref(fmt), ctypes.byref(st), _p(out)), "pack")
    return out


def unpack_page(fmt, data):
    data = np.ascontiguousarray(data, np.uint8)
    assert data.size == page_bytes(fmt)
    page = Page(fmt)
    st = page._struct()
    _ok(lib().orc_unpack_page(ctypes.byref(fmt), _p(data), ctypes.byref(st)), "unpack")
    return page


def decode_step_pages(fmt, B, H, pages, perm, q, k, v, alpha, beta, o, seed, step,
                      page_begin=0, page_end=None, plain=False):
    """fp32 step over packed pages [page_begin, page_end) in place (one
    thread); canonical order, or the plain order with plain=True."""
    if page_end is None:
        page_end = B * H
    for name, arr, dt in (("pages", pages, np.uint8), ("perm", perm, np.int32), ("q", q, np.float32),
                          ("k", k, np.float32), ("v", v, np.float32), ("alpha", alpha, np.float32),
                          ("beta", beta, np.float32), ("o", o, np.float32)):
        if arr.dtype != dt or not arr.flags["C_CONTIGUOUS"]:
            raise TypeError("%s must be a C-contiguous %s array" % (name, np.dtype(dt).name))
    fn = lib().orc_decode_step_pages_plain if plain else lib().orc_decode_step_pages
    _ok(fn(ctypes.byref(fmt), B, H, _p(pages), _p(perm), _p(q), _p(k),
           _p(v), _p(alpha), _p(beta), _p(o), int(seed), int(step),
           int(page_begin), int(page_end)), "decode_step_pages")


def f32_to_f16_rn(x):
    x = np.ascontiguousarray(x, np.float32)
    out = np.zeros(x.shape, np.uint16)
    lib().orc_f32_to_f16_rn_n(_p(x), _p(out), x.size)
    return out


def f16_to_f32(hbits):
    hbits = np.ascontiguousarray(hbits, np.uint16)
    out = np.zeros(hbits.shape, np.float32)
    lib().orc_f16_to_f32_n(_p(hbits), _p(out), hbits.size)
    return out


def div_rz(a, b):
    a = np.ascontiguousarray(a, np.float32)
    b = np.ascontiguousarray(b, np.float32)
    out = np.zeros(a.shape, np.float32)
    lib().orc_div_rz_n(_p(a), _p(b), _p(out), a.size)
    return out


def pcg4d(v):
    """pcg4d of a 4-word input (uint32 array of 4)."""
    v = np.ascontiguousarray(v, np.uint32)
    out = np.zeros(4, np.uint32)
    lib().orc_pcg4d(_p(v), _p(out))
    return out


def sr_offset(seed, step, b, h, s, j, d_v=128):
    return lib().orc_sr_offset(int(seed), int(step), int(b), int(h), int(s), int(j), int(d_v))
