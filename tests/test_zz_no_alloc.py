"""stq_calibrate_noalloc: the calibration entry point that allocates nothing.

Some callers cannot allocate device memory when they calibrate (a serving
runtime that reserved its device memory as a pool up front, code that must
not add an allocation's synchronisation to its stream, a host library given
only its inputs and outputs), so this entry point takes no workspace and uses
a fixed scratch array inside the library instead.  Called through the C ABI,
its precision map must equal stq_calibrate's, bit for bit (the map is index
work), on two calls in a row; states whose scratch need exceeds the array are
refused before anything runs.

This file is collected last so that a stopping run has already run every
other test; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from linear_attention_recurrent_delta_b200 import binding as B
from linear_attention_recurrent_delta_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _state(w):
    from linear_attention_recurrent_delta_b200 import build
    build.build()
    return B.QuantizedState(w.format, w.batch, w.heads)


@pytest.mark.parametrize("index,batch,heads", [(2, 96, 8), (3, 40, 32), (4, 33, 5)])
def test_noalloc_matches_the_workspace_entry_point_twice(index, batch, heads):
    w = W.WORKLOADS[index].resized(batch=batch, heads=heads)
    S = W.initial_state(w).cuda()
    ref = _state(w)
    B.stq_calibrate(ref.state, S)
    torch.cuda.synchronize()
    expect = ref.perm().cpu().numpy().copy()
    qs = _state(w)
    L = B.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        qs.perm().zero_()
        torch.cuda.synchronize()
        st = L.stq_calibrate_noalloc(qs.state.handle, ctypes.c_void_p(S.data_ptr()), None, stream)
        assert st == B.STQ_OK, B.stq_status_string(st)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(qs.perm().cpu().numpy(), expect, err_msg="call %d" % call)


@pytest.mark.parametrize("batch,heads", [(1, 1024), (33, 512)])
def test_noalloc_at_exactly_its_scratch_limit(batch, heads):
    """States whose scratch need is exactly the array's size (1 MiB: one
    chunk of requests x 1,024 heads, or two chunks, the second ragged, x 512
    heads) are served, and give stq_calibrate's map on two calls in a row."""
    w = W.WORKLOADS[2].resized(batch=batch, heads=heads)
    ref, qs = _state(w), _state(w)
    L = B.lib()
    assert L.stq_calibrate_workspace_bytes(qs.state.handle) == (1 << 20)
    S = W.initial_state(w, device="cuda")
    B.stq_calibrate(ref.state, S)
    for call in range(2):
        qs.perm().zero_()
        B.stq_calibrate_noalloc(qs.state, S)
        torch.cuda.synchronize()
        assert torch.equal(qs.perm(), ref.perm()), "call %d" % call


def test_noalloc_with_row_weight_matches():
    w = W.WORKLOADS[3].resized(batch=20, heads=6)
    S = W.initial_state(w).cuda()
    wgt = torch.rand(w.heads, 128, device="cuda") + 0.5
    ref, qs = _state(w), _state(w)
    B.stq_calibrate(ref.state, S, wgt)
    B.stq_calibrate_noalloc(qs.state, S, wgt)
    B.stq_calibrate_noalloc(qs.state, S, wgt)
    torch.cuda.synchronize()
    assert torch.equal(qs.perm(), ref.perm())


def test_noalloc_refuses_states_beyond_its_scratch():
    # 4096 requests x 32 heads need 4 MiB of partial scores (> 1 MiB)
    w = W.WORKLOADS[4]
    fmt = B.format_from_spec(w.format)
    L = B.lib()
    h = ctypes.c_void_p()
    fake = ctypes.c_void_p(1 << 40)          # never dereferenced: the call is refused first
    assert L.stq_state_alloc(ctypes.byref(fmt), w.batch, w.heads, fake, B.stq_state_bytes(fmt, w.batch, w.heads),
                             ctypes.byref(h)) == B.STQ_OK
    assert L.stq_calibrate_workspace_bytes(h) > (1 << 20)
    assert L.stq_calibrate_noalloc(h, ctypes.c_void_p(1 << 42), None, None) == B.STQ_ERR_BUFFER_TOO_SMALL
    L.stq_state_free(h)
    # one head past the limit: 1 MiB + 1 KiB
    w = W.WORKLOADS[2].resized(batch=1, heads=1025)
    fmt = B.format_from_spec(w.format)
    assert L.stq_state_alloc(ctypes.byref(fmt), w.batch, w.heads, fake, B.stq_state_bytes(fmt, w.batch, w.heads),
                             ctypes.byref(h)) == B.STQ_OK
    assert L.stq_calibrate_workspace_bytes(h) == (1 << 20) + 1024
    assert L.stq_calibrate_noalloc(h, ctypes.c_void_p(1 << 42), None, None) == B.STQ_ERR_BUFFER_TOO_SMALL
    L.stq_state_free(h)
