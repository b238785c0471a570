"""Shared helpers of the GPU parity tests: run the oracle and the CUDA path on
the same seeded inputs and compare them.

Rules these helpers keep: oracle inputs come from the workload generators
or from the oracle itself, never from the CUDA path; the CUDA path may be
given oracle-made pages (the same packed input for both sides).
"""
import numpy as np
import torch

import oracle as O
from linear_attention_recurrent_delta_b200 import binding as B
from linear_attention_recurrent_delta_b200 import workloads as W

BAND = 1e-5   # pre-rounding values this close to a rounding boundary may round either way


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a - b))


def oracle_quantize(w, S):
    """Oracle calibration + quantization of an fp32 state [B,H,128,128] (numpy)."""
    fmt = O.format_from_spec(w.format)
    perm = O.rank_rows(fmt, S)
    Bn, H = S.shape[:2]
    pb = O.page_bytes(fmt)
    pages = np.zeros((Bn * H, pb), np.uint8)
    for b in range(Bn):
        for h in range(H):
            pages[b * H + h] = O.pack_page(fmt, O.quantize_page(fmt, S[b, h], perm[h]))
    return fmt, perm, pages


def oracle_step(fmt, w, Bn, H, pages, perm, x, seed, step):
    """Oracle step over all pages (numpy, in a copy).  Returns (pages', o)."""
    out = pages.copy()
    o = np.zeros((Bn * H, 128), np.float32)
    arr = {k: np.ascontiguousarray(v.cpu().numpy().reshape(Bn * H, -1)) for k, v in x.items()}
    O.decode_step_pages(fmt, Bn, H, out.reshape(-1), np.ascontiguousarray(perm, np.int32), arr["q"], arr["k"],
                        arr["v"], np.ascontiguousarray(arr["alpha"].reshape(-1)),
                        np.ascontiguousarray(arr["beta"].reshape(-1)), o, seed, step)
    return out, o


def upload(qs, perm, pages):
    """Write an oracle-made precision map and pages into a QuantizedState."""
    qs.perm().copy_(torch.from_numpy(np.ascontiguousarray(perm, np.uint8)))
    qs.pages().copy_(torch.from_numpy(pages))
    torch.cuda.synchronize()


def download(qs):
    torch.cuda.synchronize()
    return qs.pages().cpu().numpy().copy()


def compare_pages(fmt, got, expect, perm=None, step_ctx=None):
    """Compare packed pages.  Returns dict(pages_equal, code_mismatch,
    band_mismatch, r_mismatch).  A code mismatch counts as a band mismatch
    only if the oracle reports the element's pre-rounding value within BAND
    of a rounding boundary (needs step_ctx = (pages_in, x, seed, step, H))."""
    res = {"pages": len(expect), "pages_equal": 0, "code_mismatch": 0, "band_mismatch": 0, "r_mismatch": 0}
    for i in range(len(expect)):
        if np.array_equal(got[i], expect[i]):
            res["pages_equal"] += 1
            continue
        pg, pe = O.unpack_page(fmt, got[i]), O.unpack_page(fmt, expect[i])
        bad = pg.code != pe.code
        res["r_mismatch"] += int(np.sum(pg.r.view(np.uint32) != pe.r.view(np.uint32)))
        if bad.any():
            res["code_mismatch"] += int(bad.sum())
            if step_ctx is not None:
                pages_in, x, seed, step, H = step_ctx
                page = O.unpack_page(fmt, pages_in[i])
                b, h = divmod(i, H)
                xs = {k: v.reshape(len(expect), -1)[i].cpu().numpy() for k, v in x.items()}
                _, _, margin = O.step_f32(fmt, page, perm[h], xs["q"], xs["k"], xs["v"], xs["alpha"],
                                          float(xs["beta"][0]), seed=seed, step=step, b=b, h=h, want_margin=True)
                res["band_mismatch"] += int(np.sum(bad & (margin < BAND)))
    return res


def make_state(w, device="cuda"):
    return B.QuantizedState(w.format, w.batch, w.heads, device=device)


def step_inputs_gpu(w, step):
    """The step's inputs generated on the CPU (the oracle's copy) and their device copy."""
    x = W.step_inputs(w, step)
    return x, {k: v.cuda() for k, v in x.items()}


# ---------------------------------------------------------------------------
# Comparison with the plain (natural key order) fp32 oracle.
#
# The pages fix no fp32 summation order, so a GPU step is compared with the
# oracle's plain evaluation (every column sum one fma chain over the key
# channels in natural order) under the rule: o and the dequantized state
# within rel-L2 1e-5; codes, packed words and row scales identical, except
# where the pre-rounding value of the plain evaluation lies within the fp32
# rounding bound of ANY summation order of a rounding boundary (or within
# 1e-5 code units of one, the fixed band).  The bound per element, in double:
#   a column sum of n = 128 products in any order is off by at most
#   g * sum_s |k_s T_sj|, g = (n + 4) u / (1 - (n + 4) u), u = 2^-24, so two
#   orders differ by at most du_j = 2 g sum_s |k_s T_sj|;
#   e = RN(v / c - u):   de_j  <= du_j (1 + 2u) + 4u (|v / c| + |u_j|);
#   T' = RN(bk e + T):   dT'_sj <= |bk_s| de_j + 4u |T'_sj|;
#   INT rows, m = max_j |T'|, inv = qmax / m, x = T' inv:
#                        dx_sj <= dT'_sj inv_s + |x_sj| (dm_s / m_s + 4u),
#                        dm_s = max_j dT'_sj;
#   FP16 rows: a differing half h must be the rounding of a value within
#   dT'_sj of the plain T' (|h - T'| <= dT' + spacing(h) / 2): near zero the
#   fp32 error of the column sums can span several binary16 steps;
# every bound doubled.  A differing INT code must move by one step.
# ---------------------------------------------------------------------------
U32 = 2.0 ** -24


def _page_values(fmt, page):
    """Element values of an unpacked page (stored order): INT codes as floats,
    FP16 rows as the floats they hold."""
    kinds = np.array([O.row_kind(fmt, s) for s in range(fmt.d_k)])
    z = page.code.astype(np.float64)
    f16 = kinds == 1
    if f16.any():
        z[f16] = O.f16_to_f32(page.code[f16].astype(np.uint16)).astype(np.float64)
    return kinds, z


def plain_step(fmt, page_in, perm_h, q, k, v, alpha, beta, seed, step, b, h):
    """The oracle's plain step from page_in (left unchanged) and the rounding
    bounds of its elements.  Returns a dict: page, o, tp, margin, dx (INT
    rows: code units), dtp (absolute, T' units), dm (per row), kinds, qmax."""
    pg = page_in.copy()
    o, tp, margin = O.step_f32(fmt, pg, perm_h, q, k, v, alpha, beta, seed=seed, step=step, b=b, h=h,
                               want_tp=True, want_margin=True, plain=True)
    perm_h = np.asarray(perm_h)
    kinds, z = _page_values(fmt, page_in)
    qmax = np.array([O.row_qmax(fmt, s) for s in range(fmt.d_k)], np.float64)
    al = np.asarray(alpha, np.float64).reshape(-1)
    al_s = al[perm_h] if fmt.gate_vector else np.full(fmt.d_k, al[0])
    r = page_in.r.astype(np.float64)
    a = np.where(kinds == 0, al_s * r, al_s)
    T = z * a[:, None]
    kp = np.asarray(k, np.float64)[perm_h]
    c = page_in.c.astype(np.float64)
    vic = np.asarray(v, np.float64) / c
    n = fmt.d_k
    g = (n + 4) * U32 / (1 - (n + 4) * U32)
    s1 = np.abs(kp[:, None] * T).sum(axis=0)
    u = (kp[:, None] * T).sum(axis=0)
    du = 2 * g * s1
    de = du * (1 + 2 * U32) + 4 * U32 * (np.abs(vic) + np.abs(u))
    bk = float(beta) * kp
    tpd = tp.astype(np.float64)
    dtp = 2 * (np.abs(bk)[:, None] * de[None, :] + 4 * U32 * np.abs(tpd))
    dm = dtp.max(axis=1)
    m = np.abs(tpd).max(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        inv = np.where(m > 0, qmax / m, 0.0)
        x = tpd * inv[:, None]
        dx = 2 * (dtp * inv[:, None] + np.abs(x) * (np.where(m > 0, dm / m, 0.0) + 4 * U32)[:, None])
    return {"page": pg, "o": o, "tp": tpd, "margin": margin, "dx": dx, "dtp": dtp, "dm": dm,
            "kinds": kinds, "qmax": qmax}


def _f16_spacing(x):
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -14)))
    return np.where(ax < 2.0 ** -14, 2.0 ** -24, 2.0 ** (e - 10))


def check_against_plain(fmt, got_page, got_o, ref, perm_h=None):
    """Compare a stepped page (unpacked) and its o with plain_step's result
    under the rule above.  Returns counts: flips (codes that differ), in_band
    (of those, within the fixed 1e-5 band), by_bound (within the derived
    bound only), outside (neither: a failure), r_diff, r_outside, o_rel,
    and state_rel when perm_h is given."""
    exp = ref["page"]
    res = {"flips": 0, "in_band": 0, "by_bound": 0, "outside": 0, "not_adjacent": 0,
           "r_diff": 0, "r_outside": 0, "o_rel": rel_l2(got_o, ref["o"])}
    bad = got_page.code != exp.code
    if bad.any():
        kinds = ref["kinds"][:, None] * np.ones_like(bad, dtype=int)
        mg = ref["margin"]
        int_el = bad & (kinds == 0)
        f16_el = bad & (kinds == 1)
        res["flips"] = int(bad.sum())
        in_band = bad & (mg < BAND)
        res["in_band"] = int(in_band.sum())
        ok_int = int_el & ~in_band & (mg <= ref["dx"])
        # an FP16 element is the binary16 rounding of its pre-rounding value:
        # a differing half is allowed if it is the rounding of some value
        # within the bound of the plain one, |h - T'| <= dT' + spacing(h) / 2
        ok_f16 = np.zeros_like(bad)
        if f16_el.any():
            hv = O.f16_to_f32(got_page.code[f16_el].astype(np.uint16)).astype(np.float64)
            dist = np.abs(hv - ref["tp"][f16_el]) - 0.5 * _f16_spacing(hv)
            ok_f16[f16_el] = dist <= ref["dtp"][f16_el]
        res["by_bound"] = int((ok_int | (ok_f16 & ~in_band)).sum())
        res["outside"] = int((bad & ~in_band & ~ok_int & ~ok_f16).sum())
        step_int = np.abs(got_page.code.astype(np.int64) - exp.code.astype(np.int64))
        # an INT code may move by one step only; an FP16 flip is bounded above
        adj = ((kinds == 0) & (step_int == 1)) | (kinds == 1)
        res["not_adjacent"] = int((bad & ~adj).sum())
    rd = got_page.r.view(np.uint32) != exp.r.view(np.uint32)
    if rd.any():
        res["r_diff"] = int(rd.sum())
        rg, re_ = got_page.r.astype(np.float64), exp.r.astype(np.float64)
        with np.errstate(divide="ignore", invalid="ignore"):
            allow = 2 * np.where(ref["qmax"] > 0, ref["dm"] / np.maximum(ref["qmax"], 1), 0) \
                + 2 * np.spacing(np.abs(exp.r)).astype(np.float64)
        res["r_outside"] = int((rd & (np.abs(rg - re_) > allow)).sum())
    if perm_h is not None:
        # the dequantized states: rel-L2 over the elements whose codes agree
        # (a flipped element differs by a whole quantization step; those are
        # the counted exceptions), and over all elements for the record
        sg = O.dequantize_page(fmt, got_page, perm_h)
        se = O.dequantize_page(fmt, exp, perm_h)
        flipped = np.zeros_like(bad)
        flipped[np.asarray(perm_h)] = bad
        res["state_rel"] = rel_l2(np.where(flipped, se, sg), se)
        res["state_rel_all"] = rel_l2(sg, se)
    return res


def assert_plain_ok(res, what=""):
    assert res["o_rel"] <= 1e-5, (what, res)
    assert res.get("state_rel", 0.0) <= 1e-5, (what, res)
    assert res["outside"] == 0 and res["not_adjacent"] == 0, (what, res)
    assert res["r_outside"] == 0, (what, res)


def add_counts(total, res):
    for k, v in res.items():
        if isinstance(v, int):
            total[k] = total.get(k, 0) + v
        else:
            total[k] = max(total.get(k, 0.0), v)
    return total


def maps_agree(fmt, S, perm_got, perm_ref, row_weight=None, rel_tie=1e-10):
    """Precision maps of the same fp32 state [B,H,128,128] from two double
    summation orders (the GPU's chunked sums, the oracle's one sequential
    sum).  A head's maps may differ only where two channels' scores at a
    group boundary lie within rel_tie of each other (both orders' rounding of
    a sum of B * 128 squares is far below 1e-10 relative).  Returns (heads
    equal, heads tied at a boundary); asserts every other head equal."""
    S = np.asarray(S, np.float64)
    sc = (S * S).sum(axis=(0, 3))                     # [H, d_k]
    if row_weight is not None:
        sc = sc * np.asarray(row_weight, np.float64)
    ends = np.cumsum([fmt.group_rows[g] for g in range(fmt.n_groups)])[:-1]
    equal, tied = 0, 0
    for h in range(sc.shape[0]):
        if np.array_equal(perm_got[h], perm_ref[h]):
            equal += 1
            continue
        srt = np.sort(sc[h])[::-1]
        gaps = [(srt[p - 1] - srt[p]) / max(srt[p - 1], 1e-300) for p in ends]
        assert gaps and min(gaps) < rel_tie, "head %d: maps differ without a tie at a group boundary" % h
        tied += 1
    return equal, tied
