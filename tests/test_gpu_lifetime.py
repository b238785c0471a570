"""GPU parity of the lifetime row weights (stq_lifetime_weights) with the
oracle, bit for bit, and of the calibration they feed: the precision map of
stq_calibrate with those weights equals the oracle's ranking with them."""
import numpy as np
import pytest
import torch

import oracle as O
from linear_attention_recurrent_delta_b200 import binding as B
from linear_attention_recurrent_delta_b200 import workloads as W

from parity_util import make_state

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from linear_attention_recurrent_delta_b200 import build
    build.build()
    B.lib()
    assert torch.cuda.is_available()


def _gate_samples(w, n):
    return torch.stack([W.step_inputs(w, 200 + t)["alpha"] for t in range(n)]).contiguous()


@pytest.mark.parametrize("name,batch,heads,n", [("stepquant4_kda", 37, 6, 9), ("stepquant6", 70, 5, 13)])
def test_weights_and_calibration_match_oracle(name, batch, heads, n):
    base = [w for w in W.WORKLOADS if w.fmt == name and w.index > 0][0]
    w = W.Workload(base.index, base.name, name, batch, heads, 2, base.gate_mu, base.gate_sigma, base.seed)
    fmt = O.format_from_spec(w.format)
    alpha = _gate_samples(w, n)
    alpha[0, 0, 0] = 1.0                                   # one gate of one: the cap
    qs = make_state(w)
    wd = torch.empty(heads, 128, device="cuda")
    B.stq_lifetime_weights(qs.state, alpha.cuda(), wd)
    torch.cuda.synchronize()
    w_ref = O.lifetime_weights(fmt, alpha.numpy())
    assert np.array_equal(wd.cpu().numpy().view(np.uint32), w_ref.view(np.uint32))
    S = W.initial_state(w)
    B.stq_calibrate(qs.state, S.cuda(), row_weight=wd)
    torch.cuda.synchronize()
    assert np.array_equal(qs.perm().cpu().numpy(), O.rank_rows(fmt, S.numpy(), row_weight=w_ref))
