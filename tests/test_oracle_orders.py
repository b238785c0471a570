"""The kernel's canonical fp32 summation order against the plain one.

The pages fix no fp32 evaluation order.  The oracle keeps two: the plain one
(every column sum one fma chain over the key channels in natural order, the
definition written left to right) and the canonical one (the decode kernel's
slices, halves and tree), which the GPU reproduces bit for bit.  Here the
canonical step is compared with the plain step under the same rule the GPU
is held to against the plain oracle: o and the dequantized state within
rel-L2 1e-5; codes and row scales identical except where the plain
pre-rounding value lies within the fixed 1e-5 band or within the fp32
rounding bound of any summation order of a rounding boundary.  So the
canonical order is shown to be one fair fp32 evaluation of the definition,
and the flips it makes against the plain order are counted per format.
A planted mistake (a wrong sign in the update) must fail the same rule.
"""
import numpy as np
import pytest

import oracle as O
from linear_attention_recurrent_delta_b200 import workloads as W

from parity_util import add_counts, assert_plain_ok, check_against_plain, oracle_quantize, plain_step

FLIPS = {}


def _case(index, batch=2, steps=3):
    w = W.WORKLOADS[index].resized(batch=batch)
    S = W.initial_state(w).numpy()
    fmt, perm, pages = oracle_quantize(w, S)
    return w, fmt, perm, pages


@pytest.mark.parametrize("index", [1, 2, 3, 4])
def test_canonical_order_is_within_the_plain_rounding_band(index):
    w, fmt, perm, pages = _case(index)
    seed = W.sr_seed(w)
    total = {}
    for step in range(3):
        x = W.step_inputs(w, step)
        xs = {k: v.numpy().reshape(w.pages, -1) for k, v in x.items()}
        for i in range(w.pages):
            b, h = divmod(i, w.heads)
            page = O.unpack_page(fmt, pages[i])
            args = (xs["q"][i], xs["k"][i], xs["v"][i], xs["alpha"][i], float(xs["beta"][i][0]))
            ref = plain_step(fmt, page, perm[h], *args, seed, step, b, h)
            got = page.copy()
            o, _, _ = O.step_f32(fmt, got, perm[h], *args, seed=seed, step=step, b=b, h=h)
            res = check_against_plain(fmt, got, o, ref, perm[h])
            assert_plain_ok(res, (w.name, step, i))
            add_counts(total, res)
            pages[i] = O.pack_page(fmt, got)
    FLIPS[w.name] = total
    print("\n%s: %d pages x 3 steps, code flips %d (in the 1e-5 band %d, by the order bound %d), "
          "row scales differing %d, max o rel-L2 %.2e" % (w.name, w.pages, total["flips"], total["in_band"],
                                                          total["by_bound"], total["r_diff"], total["o_rel"]))


def test_a_planted_sign_error_fails_the_rule():
    """The rule has teeth: the plain step's page with the update's sign
    flipped (T - bk e instead of T + bk e, made here on the CPU) is rejected."""
    w, fmt, perm, pages = _case(2, batch=1)
    x = W.step_inputs(w, 0)
    xs = {k: v.numpy().reshape(w.pages, -1) for k, v in x.items()}
    i, h = 3, 3
    page = O.unpack_page(fmt, pages[i])
    q, k, v, a, beta = xs["q"][i], xs["k"][i], xs["v"][i], xs["alpha"][i], float(xs["beta"][i][0])
    ref = plain_step(fmt, page, perm[h], q, k, v, a, beta, 0, 0, 0, h)
    bad = page.copy()
    o_bad, _, _ = O.step_f32(fmt, bad, perm[h], q, k, v, a, -beta, plain=True)   # -beta: T - bk e
    res = check_against_plain(fmt, bad, o_bad, ref, perm[h])
    assert res["outside"] > 0 or res["o_rel"] > 1e-5
