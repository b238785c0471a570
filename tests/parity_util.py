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
