"""Thin ctypes binding over the C ABI in include/stq.h (``libstq.so``).

Argument marshalling only: every step of the path runs in the library's
kernels.  Tensors are torch tensors (device memory and streams come from
torch); functions keep the C names.  Loading fails loudly when the library
has not been built -- there is no fallback of any kind.
"""
import ctypes
import os
from ctypes import c_int, c_size_t, c_uint32, c_uint64, c_void_p, c_char_p, POINTER

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libstq.so")
MAX_GROUPS = 8

STQ_OK, STQ_ERR_INVALID_ARG, STQ_ERR_UNSUPPORTED, STQ_ERR_BUFFER_TOO_SMALL, \
    STQ_ERR_MISALIGNED, STQ_ERR_CUDA, STQ_ERR_DEVICE_TIMEOUT = range(7)
STQ_WINDOW_MAX = 16   # steps in a window at most (include/stq.h)
STQ_INT, STQ_FP16 = 0, 1


class StqFormat(ctypes.Structure):
    _fields_ = [("d_k", c_int), ("d_v", c_int), ("n_groups", c_int),
                ("group_rows", c_int * MAX_GROUPS), ("group_kind", c_int * MAX_GROUPS),
                ("group_bits", c_int * MAX_GROUPS), ("col_scales", c_int),
                ("stochastic", c_int), ("gate_vector", c_int)]


class StqError(RuntimeError):
    def __init__(self, status, what):
        super().__init__("%s: %s (%d)" % (what, stq_status_string(status), status))
        self.status = status


_lib = None


def lib():
    """Load libstq.so (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libstq.so is not built (%s); run __graft_entry__.build() or "
                           "python linear_attention_recurrent_delta_b200/build.py" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    P = c_void_p
    sigs = {
        "stq_page_bytes": (c_size_t, [P]),
        "stq_state_bytes": (c_size_t, [P, c_int, c_int]),
        "stq_state_alloc": (c_int, [P, c_int, c_int, P, c_size_t, POINTER(c_void_p)]),
        "stq_state_free": (None, [P]),
        "stq_state_layout": (c_int, [P, POINTER(c_size_t), POINTER(c_size_t), POINTER(c_size_t),
                                     POINTER(c_size_t)]),
        "stq_calibrate_workspace_bytes": (c_size_t, [P]),
        "stq_calibrate": (c_int, [P, P, P, P, c_size_t, P]),
        "stq_calibrate_noalloc": (c_int, [P, P, P, P]),
        "stq_quantize_state": (c_int, [P, P, P]),
        "stq_quantize_state_fit": (c_int, [P, P, P, c_int, P]),
        "stq_decode_step": (c_int, [P, P, P, P, P, P, P, c_uint64, c_uint32, P]),
        "stq_decode_step_slots": (c_int, [P, P, c_int, P, P, P, P, P, P, c_uint64, c_uint32, P]),
        "stq_request_pages": (c_int, [P, c_int, POINTER(c_size_t), POINTER(c_size_t)]),
        "stq_window_buffer_bytes": (c_size_t, [P, c_int]),
        "stq_window_step": (c_int, [P, P, c_size_t, c_int, c_int, c_int, P, P, P, P, P, P, c_uint64, c_uint32, P]),
        "stq_lifetime_weights": (c_int, [P, P, c_int, P, P]),
        "stq_prefill": (c_int, [P, c_int, P, P, P, P, P, P, P, c_uint64, c_uint32, P]),
        "stq_prefill_chunked": (c_int, [P, c_int, P, P, P, P, P, P, P, c_uint64, c_uint32, P]),
        "stq_decode_io_bytes": (c_size_t, [P]),
        "stq_decode_step_host": (c_int, [P, P, P, P, P, P, P, P, c_size_t, c_uint64, c_uint32, P]),
        "stq_decode_steps_host": (c_int, [P, c_int, P, P, P, P, P, P, P, c_size_t, c_uint64, c_uint32, P]),
        "stq_dequantize_state": (c_int, [P, P, P]),
        "stq_device_status": (c_int, [P, P, c_int]),
        "stq_set_wait_limit": (c_int, [P, c_uint64, c_int]),
        "stq_status_string": (c_char_p, [c_int]),
        "stq_version": (c_int, []),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def stq_status_string(status):
    return lib().stq_status_string(int(status)).decode()


def stq_version():
    return lib().stq_version()


def _check(status, what):
    if status != STQ_OK:
        raise StqError(status, what)


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def make_format(groups, col_scales=False, stochastic=False, gate_vector=False, d_k=128, d_v=128):
    """groups: list of (rows, kind, bits), kind "int" or "fp16"."""
    f = StqFormat()
    f.d_k, f.d_v, f.n_groups = d_k, d_v, len(groups)
    for i, (rows, kind, bits) in enumerate(groups):
        f.group_rows[i] = rows
        f.group_kind[i] = {"int": STQ_INT, "fp16": STQ_FP16}[kind]
        f.group_bits[i] = bits if kind == "int" else 0
    f.col_scales, f.stochastic, f.gate_vector = int(col_scales), int(stochastic), int(gate_vector)
    return f


def format_from_spec(spec):
    return make_format(spec["groups"], spec["col_scales"], spec["stochastic"], spec["gate_vector"])


def stq_page_bytes(fmt):
    return lib().stq_page_bytes(ctypes.byref(fmt))


def stq_state_bytes(fmt, batch, heads):
    return lib().stq_state_bytes(ctypes.byref(fmt), batch, heads)


class State:
    """Host descriptor bound to a device buffer (kept alive here)."""

    def __init__(self, handle, fmt, batch, heads, buf):
        self.handle, self.fmt, self.batch, self.heads, self.buf = handle, fmt, batch, heads, buf

    def __del__(self):
        if getattr(self, "handle", None) and _lib is not None:
            _lib.stq_state_free(self.handle)
            self.handle = None


def stq_state_alloc(fmt, batch, heads, buf, nbytes=None):
    """Bind ``buf`` (a device tensor) as the state of ``batch`` x ``heads`` pages."""
    h = c_void_p()
    n = buf.numel() * buf.element_size() if nbytes is None else nbytes
    _check(lib().stq_state_alloc(ctypes.byref(fmt), batch, heads, _ptr(buf), n, ctypes.byref(h)),
           "stq_state_alloc")
    return State(h, fmt, batch, heads, buf)


def stq_state_layout(state):
    vals = [c_size_t() for _ in range(4)]
    _check(lib().stq_state_layout(state.handle, *[ctypes.byref(v) for v in vals]), "stq_state_layout")
    return dict(zip(("page_bytes", "perm_offset", "pages_offset", "status_offset"), (v.value for v in vals)))


def stq_calibrate_workspace_bytes(state):
    return lib().stq_calibrate_workspace_bytes(state.handle)


def stq_calibrate(state, S, row_weight=None, workspace=None, stream=None):
    import torch
    need = stq_calibrate_workspace_bytes(state)
    if workspace is None:
        workspace = torch.empty(max(need, 8), dtype=torch.uint8, device=S.device)
    _check(lib().stq_calibrate(state.handle, _ptr(S), _ptr(row_weight), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream)), "stq_calibrate")


def stq_calibrate_noalloc(state, S, row_weight=None, stream=None):
    """stq_calibrate with the library's fixed scratch (no workspace, no allocation)."""
    _check(lib().stq_calibrate_noalloc(state.handle, _ptr(S), _ptr(row_weight), _stream(stream)),
           "stq_calibrate_noalloc")


def stq_quantize_state(state, S, stream=None):
    _check(lib().stq_quantize_state(state.handle, _ptr(S), _stream(stream)), "stq_quantize_state")


def stq_quantize_state_fit(state, S, row_impact=None, iters=4, stream=None):
    """Quantize with jointly fitted row and column scales (row_impact: [H, 128] or None)."""
    _check(lib().stq_quantize_state_fit(state.handle, _ptr(S), _ptr(row_impact), int(iters), _stream(stream)),
           "stq_quantize_state_fit")


def stq_decode_step(state, q, k, v, alpha, beta, o, seed=0, step=0, stream=None):
    _check(lib().stq_decode_step(state.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(o),
                                 int(seed), int(step), _stream(stream)), "stq_decode_step")


def stq_decode_step_slots(state, slots, q, k, v, alpha, beta, o, seed=0, step=0, stream=None):
    """Step the requests in state slots ``slots`` (int32 device tensor, one per input row)."""
    _check(lib().stq_decode_step_slots(state.handle, _ptr(slots), int(slots.numel()), _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(alpha), _ptr(beta), _ptr(o), int(seed), int(step), _stream(stream)),
           "stq_decode_step_slots")


def stq_request_pages(state, slot):
    """(byte offset, bytes) of the pages of the request in ``slot`` inside the state buffer."""
    off, n = c_size_t(), c_size_t()
    _check(lib().stq_request_pages(state.handle, int(slot), ctypes.byref(off), ctypes.byref(n)), "stq_request_pages")
    return off.value, n.value


def stq_window_buffer_bytes(state, window):
    return lib().stq_window_buffer_bytes(state.handle, int(window))


def stq_window_step(state, buf, window, t, commit, q, k, v, alpha, beta, o, seed=0, step=0, stream=None):
    """Step t of a window of ``window`` steps (``buf``: uint8 device tensor of
    stq_window_buffer_bytes); ``commit`` requantizes the pages."""
    _check(lib().stq_window_step(state.handle, _ptr(buf), buf.numel() * buf.element_size(), int(window), int(t),
                                 int(bool(commit)), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(o),
                                 int(seed), int(step), _stream(stream)), "stq_window_step")


def stq_lifetime_weights(state, alpha, row_weight, stream=None):
    """Row weights [H, 128] from gate samples alpha [n_samples, B, H(, 128)]."""
    _check(lib().stq_lifetime_weights(state.handle, _ptr(alpha), int(alpha.shape[0]), _ptr(row_weight),
                                      _stream(stream)), "stq_lifetime_weights")


def stq_prefill(state, q, k, v, alpha, beta, o, S_out=None, seed=0, step=0, stream=None):
    """A prompt of L = q.shape[0] tokens through every page (q, k, v, o: [L, B, H, 128])."""
    _check(lib().stq_prefill(state.handle, int(q.shape[0]), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                             _ptr(o), _ptr(S_out), int(seed), int(step), _stream(stream)), "stq_prefill")


def stq_prefill_chunked(state, q, k, v, alpha, beta, o, S_out=None, seed=0, step=0, stream=None):
    """The same prompt in chunkwise form on the tensor cores (scalar-gate formats)."""
    _check(lib().stq_prefill_chunked(state.handle, int(q.shape[0]), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                     _ptr(beta), _ptr(o), _ptr(S_out), int(seed), int(step), _stream(stream)),
           "stq_prefill_chunked")


def stq_decode_io_bytes(state):
    return lib().stq_decode_io_bytes(state.handle)


def stq_decode_step_host(state, hq, hk, hv, halpha, hbeta, ho, io, seed=0, step=0, stream=None):
    _check(lib().stq_decode_step_host(state.handle, _ptr(hq), _ptr(hk), _ptr(hv), _ptr(halpha), _ptr(hbeta),
                                      _ptr(ho), _ptr(io), io.numel() * io.element_size(), int(seed),
                                      int(step), _stream(stream)), "stq_decode_step_host")


def stq_decode_steps_host(state, hq, hk, hv, halpha, hbeta, ho, io, seed=0, step=0, stream=None):
    """hq.shape[0] steps from pinned host tensors [n, B, H, ...], copies overlapped with the steps."""
    _check(lib().stq_decode_steps_host(state.handle, int(hq.shape[0]), _ptr(hq), _ptr(hk), _ptr(hv), _ptr(halpha),
                                       _ptr(hbeta), _ptr(ho), _ptr(io), io.numel() * io.element_size(), int(seed),
                                       int(step), _stream(stream)), "stq_decode_steps_host")


def stq_dequantize_state(state, S, stream=None):
    _check(lib().stq_dequantize_state(state.handle, _ptr(S), _stream(stream)), "stq_dequantize_state")


def stq_device_status(state, stream=None, clear=False):
    return lib().stq_device_status(state.handle, _stream(stream), int(clear))


def stq_set_wait_limit(state, limit_ns, stall_first_wait=False):
    _check(lib().stq_set_wait_limit(state.handle, int(limit_ns), int(stall_first_wait)), "stq_set_wait_limit")


class QuantizedState:
    """A quantized recurrent state of ``batch`` x ``heads`` pages on one GPU.

    Owns its device buffer (a torch uint8 tensor).  ``calibrate_and_quantize``
    builds the precision map and the packed pages from an fp32 state
    [B, H, 128, 128]; ``step`` runs one decode step in place and returns o.
    """

    def __init__(self, spec, batch, heads, device="cuda"):
        import torch
        self.spec = spec
        self.fmt = format_from_spec(spec)
        nbytes = stq_state_bytes(self.fmt, batch, heads)
        if nbytes == 0:
            raise StqError(STQ_ERR_UNSUPPORTED, "stq_state_bytes")
        self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 256
        self.view = self.buf[off:off + nbytes]
        self.state = stq_state_alloc(self.fmt, batch, heads, self.view, nbytes)
        self.batch, self.heads = batch, heads
        self.layout = stq_state_layout(self.state)
        # a fresh buffer holds whatever the allocator left there: clear the
        # header (status word) and the precision map
        self.view[:self.layout["pages_offset"]].zero_()

    def calibrate_and_quantize(self, S, row_weight=None, stream=None):
        stq_calibrate(self.state, S, row_weight, stream=stream)
        stq_quantize_state(self.state, S, stream=stream)

    def step(self, q, k, v, alpha, beta, o=None, seed=0, step=0, stream=None):
        import torch
        if o is None:
            o = torch.empty_like(q)
        stq_decode_step(self.state, q, k, v, alpha, beta, o, seed, step, stream)
        return o

    def dequantize(self, stream=None):
        import torch
        S = torch.empty(self.batch, self.heads, 128, 128, dtype=torch.float32, device=self.buf.device)
        stq_dequantize_state(self.state, S, stream)
        return S

    def pages(self):
        """Device view of the packed pages, [B*H, page_bytes] uint8."""
        L = self.layout
        n = self.batch * self.heads
        return self.view[L["pages_offset"]:L["pages_offset"] + n * L["page_bytes"]].view(n, L["page_bytes"])

    def perm(self):
        """Device view of the precision map, [H, 128] uint8."""
        L = self.layout
        return self.view[L["perm_offset"]:L["perm_offset"] + self.heads * 128].view(self.heads, 128)
