"""GPU parity of the lifetime row weights (stq_lifetime_weights) with the
oracle, and of the calibration they feed.

The mean gate is a double sum of n_samples x B gates: the oracle adds them in
one sequential chain, the kernel in parallel slices, so the two doubles
differ by at most (n B) 2^-53 relative, and 1 / (1 - mean) by that times
mean / (1 - mean).  Below 2^-24 that leaves the float result within one ulp
of the oracle's (the test checks the bound holds, then the ulp), and equal
unless the double lies that close to a float rounding boundary (counted).
The precision map with those weights equals the oracle's except at a tie of
scores (within the weights' ulp) at a group boundary."""
import numpy as np
import pytest
import torch

import oracle as O
from linear_attention_recurrent_delta_b200 import binding as B
from linear_attention_recurrent_delta_b200 import workloads as W

from parity_util import make_state, maps_agree

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
    got = wd.cpu().numpy()
    # the order bound: (n B) 2^-53 relative on the mean, amplified by mean / (1 - mean)
    a = alpha.numpy().astype(np.float64)
    mean = a.reshape(n * batch, heads, -1).mean(axis=0).reshape(heads, -1)
    if not fmt.gate_vector:
        mean = np.repeat(mean, 128, axis=1)
    gap = np.maximum(1 - mean, 2.0 ** -24)
    bound = n * batch * 2.0 ** -53 * (1 + mean / gap)
    assert bound.max() < 2.0 ** -24
    ulp = np.spacing(np.abs(w_ref)).astype(np.float64)
    diff = np.abs(got.astype(np.float64) - w_ref.astype(np.float64))
    assert np.all(diff <= ulp), diff.max()
    off = int(np.sum(got.view(np.uint32) != w_ref.view(np.uint32)))
    print("lifetime weights: %d of %d one ulp off the oracle's" % (off, got.size))
    S = W.initial_state(w)
    B.stq_calibrate(qs.state, S.cuda(), row_weight=wd)
    torch.cuda.synchronize()
    perm_ref = O.rank_rows(fmt, S.numpy(), row_weight=w_ref)
    equal, tied = maps_agree(fmt, S.numpy(), qs.perm().cpu().numpy(), perm_ref, row_weight=w_ref, rel_tie=2.0 ** -21)
    print("calibration with the weights: %d heads equal, %d tied at a group boundary" % (equal, tied))
