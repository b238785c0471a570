"""Seeded synthetic workloads for the quantized decode step.

This module holds the workload descriptions and the seeded input generators,
and nothing of the method's arithmetic: no quantization, no packing, no
update.  It is the one module that both the CUDA path (bench, tests) and the
CPU oracle's callers use, so that both sides see the same inputs.

Distributions (the same for every configuration, sizes differ):
  * initial state  S[b,h,i,j] = N(0,1) * exp(N(0,1))_row[h,i] * exp(N(0,1))_col[h,j]
    (log-normal row and column magnitudes, drawn per head and shared by the
    requests of the batch, so the state shows the row and column outliers of
    the STEPQuant page's Fig. 5 / Figure B2);
  * per step  q, k ~ N(0,1)^128, each L2-normalised;  v ~ N(0,1)^128;
  * GDN gate  alpha = exp(-softplus(a)), a ~ N(-4, 1), one per (request, head);
  * KDA gate  alpha_i = exp(-softplus(a_i)), a_i ~ N(-4, 1.5), per key channel;
  * beta = sigmoid(N(0,1)).
Generation uses torch generators on the requested device; the same seed on
the same device gives the same tensors.
"""
from dataclasses import dataclass

import torch

D = 128

# Row-group formats.  groups: (rows, kind, bits), widest first.
FORMATS = {
    # STEPQuant-style nominal 6-bit: 32 x INT8 / 64 x INT6 / 32 x INT4, row and column scales
    "stepquant6": {"groups": [(32, "int", 8), (64, "int", 6), (32, "int", 4)],
                   "col_scales": True, "stochastic": False, "gate_vector": False},
    # uniform per-row INT8 (column scale fixed at 1)
    "int8row": {"groups": [(128, "int", 8)],
                "col_scales": False, "stochastic": False, "gate_vector": False},
    # STEPQuant-style nominal 4-bit with a KDA per-key-channel gate
    "stepquant4_kda": {"groups": [(16, "int", 8), (48, "int", 4), (64, "int", 3)],
                       "col_scales": True, "stochastic": False, "gate_vector": True},
    # DAMP-style: 16 key rows FP16, 112 rows INT8 with stochastic rounding, row scales only
    "damp": {"groups": [(16, "fp16", 0), (112, "int", 8)],
             "col_scales": False, "stochastic": True, "gate_vector": False},
}


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    fmt: str
    batch: int
    heads: int
    steps: int
    gate_mu: float = -4.0
    gate_sigma: float = 1.0
    seed: int = 0

    @property
    def pages(self) -> int:
        return self.batch * self.heads

    @property
    def format(self) -> dict:
        return FORMATS[self.fmt]

    def resized(self, batch=None, heads=None, steps=None):
        return Workload(self.index, self.name, self.fmt, batch or self.batch, heads or self.heads,
                        steps or self.steps, self.gate_mu, self.gate_sigma, self.seed)


def _wl(index, name, fmt, batch, heads, steps, gate_sigma=1.0):
    return Workload(index, name, fmt, batch, heads, steps, -4.0, gate_sigma, 0x57E90000 + index)


WORKLOADS = [
    _wl(0, "tiny-gdn-stepquant6", "stepquant6", 1, 4, 64),
    _wl(1, "int8row-gdn", "int8row", 256, 32, 128),
    _wl(2, "stepquant6-gdn", "stepquant6", 1024, 32, 64),
    _wl(3, "stepquant4-kda", "stepquant4_kda", 2048, 32, 64, gate_sigma=1.5),
    _wl(4, "damp-gdn", "damp", 4096, 32, 32),
]


def _gen(device, *key):
    g = torch.Generator(device=device)
    s = 0
    for x in key:
        s = (s * 1000003 + int(x)) & 0x7FFFFFFFFFFFFFFF
    g.manual_seed(s)
    return g


def initial_state(w: Workload, device="cpu", batch=None):
    """Unquantized fp32 state [B, H, 128, 128] (natural key order)."""
    B = batch or w.batch
    g = _gen(device, w.seed, 1)
    row = torch.exp(torch.randn(w.heads, D, 1, generator=g, device=device))
    col = torch.exp(torch.randn(w.heads, 1, D, generator=g, device=device))
    S = torch.empty(B, w.heads, D, D, device=device)
    chunk = max(1, (1 << 28) // (w.heads * D * D * 4))
    for b0 in range(0, B, chunk):
        b1 = min(B, b0 + chunk)
        gb = _gen(device, w.seed, 2, b0)
        S[b0:b1] = torch.randn(b1 - b0, w.heads, D, D, generator=gb, device=device) * row * col
    return S


def step_inputs(w: Workload, step: int, device="cpu", batch=None):
    """Inputs of one decode step: dict of q, k, v [B,H,128], alpha [B,H] or
    [B,H,128], beta [B,H] (all fp32, contiguous)."""
    B = batch or w.batch
    H = w.heads
    g = _gen(device, w.seed, 3, step)
    q = torch.randn(B, H, D, generator=g, device=device)
    k = torch.randn(B, H, D, generator=g, device=device)
    v = torch.randn(B, H, D, generator=g, device=device)
    q = q / torch.linalg.vector_norm(q, dim=-1, keepdim=True)
    k = k / torch.linalg.vector_norm(k, dim=-1, keepdim=True)
    gate_shape = (B, H, D) if w.format["gate_vector"] else (B, H)
    a = w.gate_mu + w.gate_sigma * torch.randn(gate_shape, generator=g, device=device)
    alpha = torch.exp(-torch.nn.functional.softplus(a))
    beta = torch.sigmoid(torch.randn(B, H, generator=g, device=device))
    return {"q": q.contiguous(), "k": k.contiguous(), "v": v.contiguous(),
            "alpha": alpha.contiguous(), "beta": beta.contiguous()}


def sr_seed(w: Workload) -> int:
    """64-bit seed of the stochastic-rounding generator for a workload."""
    return (0x5EED0000 + w.index) * 0x100000001
