"""Failure detection without a GPU fault.

Every device-side wait of the decode kernel is bounded.  The test hook makes
the first pipeline wait of each CTA wait on a barrier that nothing ever
completes; after the (short) limit the kernel records a timeout in the
state's status word, lets its in-flight copies land, and returns.  The host
reads STQ_ERR_DEVICE_TIMEOUT, and the context stays usable: the next step
runs normally and matches the oracle.
"""
import numpy as np
import pytest
import torch

from linear_attention_recurrent_delta_b200 import binding as B
from linear_attention_recurrent_delta_b200 import workloads as W

from parity_util import download, make_state, oracle_quantize, oracle_step, step_inputs_gpu, upload

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_survives():
    from linear_attention_recurrent_delta_b200 import build
    build.build()
    w = W.WORKLOADS[2].resized(batch=3, heads=4, steps=1)
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    qs = make_state(w)
    upload(qs, perm, pages)
    x, xd = step_inputs_gpu(w, 0)
    B.stq_set_wait_limit(qs.state, 20_000_000, stall_first_wait=True)   # 20 ms
    qs.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"])
    assert B.stq_device_status(qs.state, clear=True) == B.STQ_ERR_DEVICE_TIMEOUT
    assert np.array_equal(download(qs), pages)          # nothing was written
    assert B.stq_device_status(qs.state) == B.STQ_OK     # cleared
    B.stq_set_wait_limit(qs.state, 0, stall_first_wait=False)
    o = qs.step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta"])
    assert B.stq_device_status(qs.state) == B.STQ_OK
    expect, o_ref = oracle_step(fmt, w, w.batch, w.heads, pages, perm, x, 0, 0)
    assert np.array_equal(download(qs), expect)
    assert np.array_equal(o.cpu().numpy().reshape(w.pages, 128), o_ref)
    torch.cuda.synchronize()
