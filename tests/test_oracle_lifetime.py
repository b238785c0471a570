"""Pins of the oracle's lifetime weights (orc_lifetime_weights), the row
weight of the calibration that gives long-lived key channels more bits.

* exact cases: a constant gate alpha gives 1 / (1 - alpha) for alpha = 0,
  1/2, 3/4, 7/8 (exact in binary); a gate of one is capped at 2^24;
* the mean runs over samples and requests: samples {1/2, 1} give 4;
* layout: one (head, channel) with another gate changes that weight only
  (KDA), a GDN head's gate sets all of its channels;
* with equal row energies the ranking puts the longest-lived channels in the
  widest group.
"""
import numpy as np
import pytest

import oracle as O
from linear_attention_recurrent_delta_b200 import workloads as W

KDA = O.format_from_spec(W.FORMATS["stepquant4_kda"])
GDN = O.format_from_spec(W.FORMATS["stepquant6"])


@pytest.mark.parametrize("a,w", [(0.0, 1.0), (0.5, 2.0), (0.75, 4.0), (0.875, 8.0), (1.0, 2.0**24)])
def test_constant_gate(a, w):
    alpha = np.full((5, 3, 2, 128), a, np.float32)
    assert np.all(O.lifetime_weights(KDA, alpha) == np.float32(w))


def test_mean_over_samples_and_requests():
    alpha = np.full((4, 6, 2, 128), 0.5, np.float32)
    alpha[::2, :, 0, 9] = 1.0                       # half the samples of channel 9 (head 0) keep everything
    alpha[:, 3:, 1, 40] = 1.0                       # half the requests of channel 40 (head 1) likewise
    w = O.lifetime_weights(KDA, alpha)
    assert w[0, 9] == 4.0 and w[1, 40] == 4.0
    others = np.ones_like(w, bool)
    others[0, 9] = others[1, 40] = False
    assert np.all(w[others] == 2.0)


def test_layout_kda_and_gdn():
    rng = np.random.default_rng(3)
    alpha = np.full((2, 3, 4, 128), 0.5, np.float32)
    h, k = 2, 77
    alpha[:, :, h, k] = 0.875
    w = O.lifetime_weights(KDA, alpha)
    assert w[h, k] == 8.0 and np.count_nonzero(w != 2.0) == 1
    g = (1 / (1 + np.exp(-rng.normal(2, 1, size=(7, 5, 4))))).astype(np.float32)   # GDN: [samples, B, H]
    wg = O.lifetime_weights(GDN, g)
    for hh in range(4):
        assert np.all(wg[hh] == wg[hh, 0])
    assert len(set(wg[:, 0].tolist())) == 4
    # monotone in the mean gate
    order = np.argsort(g.astype(np.float64).mean(axis=(0, 1)))
    assert np.all(np.diff(wg[order, 0]) > 0)


def test_long_lived_channels_rank_first():
    """Equal row energies: the ranking follows the weights alone, so the
    channels with the longest-lived gates fill the widest group."""
    rng = np.random.default_rng(8)
    S = np.ones((2, 1, 128, 128), np.float32) * rng.choice([-1.0, 1.0], size=(2, 1, 128, 128)).astype(np.float32)
    alpha = np.full((3, 2, 1, 128), 0.5, np.float32)
    longlived = rng.permutation(128)[:16]
    alpha[:, :, 0, longlived] = 0.96875             # 1 / (1 - alpha) = 32
    w = O.lifetime_weights(KDA, alpha)
    perm = O.rank_rows(KDA, S, row_weight=w)[0]
    first = KDA.group_rows[0]
    assert set(perm[:first].tolist()) == set(sorted(longlived.tolist())[:first])
    without = O.rank_rows(KDA, S)[0]
    assert list(without[:first]) == list(range(first))   # ties without weights: lower channel first
