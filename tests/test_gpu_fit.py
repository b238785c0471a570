"""GPU parity of the joint scale fit (stq_quantize_state_fit) with the oracle.

Both sides run the same double operations in the same order (codes by one
correctly rounded double division, sums j ascending per row and kappa
ascending per column, each scale rounded to float once per update), so the
packed pages must agree bit for bit.  Every format, equal and per-row impact
weights, 0, 1 and 4 rounds, at 37 x 9 pages (more pages than resident CTAs,
ragged tail); a zero row and a zero column in the state.  The fit must also
lower the impact-weighted reconstruction error against the absmax pages.
"""
import numpy as np
import pytest
import torch

import oracle as O
from linear_attention_recurrent_delta_b200 import binding as B
from linear_attention_recurrent_delta_b200 import workloads as W

from parity_util import download, make_state

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from linear_attention_recurrent_delta_b200 import build
    build.build()
    B.lib()
    assert torch.cuda.is_available()


def _small(name, batch=37, heads=9):
    w = [x for x in W.WORKLOADS if x.fmt == name and x.index > 0][0]
    return w.resized(batch=batch, heads=heads, steps=2)


@pytest.mark.parametrize("iters", [0, 1, 4])
@pytest.mark.parametrize("weighted", [False, True])
@pytest.mark.parametrize("name", list(W.FORMATS))
def test_fit_matches_oracle(name, weighted, iters):
    w = _small(name)
    S = W.initial_state(w)
    S[0, 1, 5] = 0.0          # a zero key row
    S[2, 3, :, 9] = 0.0       # a zero value column
    fmt = O.format_from_spec(w.format)
    perm = O.rank_rows(fmt, S.numpy())
    imp = None
    if weighted:
        imp = torch.rand(w.heads, 128, generator=torch.Generator().manual_seed(7)) + 0.25
    qs = make_state(w)
    qs.perm().copy_(torch.from_numpy(np.ascontiguousarray(perm, np.uint8)))
    B.stq_quantize_state_fit(qs.state, S.cuda(), None if imp is None else imp.cuda(), iters)
    got = download(qs)
    assert B.stq_device_status(qs.state) == B.STQ_OK
    Sn = S.numpy()
    gain = []
    for i in range(w.pages):
        b, h = divmod(i, w.heads)
        page, err = O.quantize_page_fit(fmt, Sn[b, h], perm[h], None if imp is None else imp[h].numpy(), iters)
        expect = O.pack_page(fmt, page)
        assert np.array_equal(got[i], expect), "page %d (%d rounds)" % (i, iters)
        gain.append(1 - err[-1] / max(err[0], 1e-300))
    print("\n%s, %d rounds%s: mean reduction of the weighted error %.3f" %
          (name, iters, " (impact weights)" if weighted else "", float(np.mean(gain))))


def test_fit_argument_errors():
    w = _small("stepquant6", batch=2, heads=2)
    qs = make_state(w)
    S = torch.zeros(w.batch, w.heads, 128, 128, device="cuda")
    L = B.lib()
    assert L.stq_quantize_state_fit(qs.state.handle, B._ptr(S), None, -1, None) == B.STQ_ERR_INVALID_ARG
    assert L.stq_quantize_state_fit(qs.state.handle, B._ptr(S), None, 17, None) == B.STQ_ERR_INVALID_ARG
    assert L.stq_quantize_state_fit(qs.state.handle, None, None, 2, None) == B.STQ_ERR_INVALID_ARG
    imp = torch.zeros(w.heads * 128 + 1, device="cuda")
    assert L.stq_quantize_state_fit(qs.state.handle, B._ptr(S), imp[1:].data_ptr() + 1 if False else
                                    imp.data_ptr() + 2, 2, None) == B.STQ_ERR_MISALIGNED
    # the state's own bytes as the impact weights: refused
    assert L.stq_quantize_state_fit(qs.state.handle, B._ptr(S), qs.pages().data_ptr(), 2, None) == \
        B.STQ_ERR_INVALID_ARG
