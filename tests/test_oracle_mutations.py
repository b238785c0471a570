"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake (a dropped term, a wrong sign, a wrong index, a
transposed operand, a wrong constant) in a temporary copy of the oracle
source, builds it, and runs the other oracle pin files against it: the run
must fail.  The planted copies live only in a temporary directory on the CPU.
"""
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "stq_oracle.cpp")
HDR = os.path.join(ROOT, "oracle", "stq_oracle.h")
PIN_FILES = ["tests/test_oracle_scalars.py", "tests/test_oracle_format.py",
             "tests/test_oracle_quantize.py", "tests/test_oracle_step.py", "tests/test_oracle_window.py",
             "tests/test_oracle_prefill.py", "tests/test_oracle_lifetime.py", "tests/test_oracle_fit.py",
             "tests/test_oracle_chunked.py"]

MUTANTS = {
    "error sign": ("e[j] = v[j] * ic[j] - u[j];", "e[j] = v[j] * ic[j] + u[j];"),
    "key index not permuted": ("float bk = beta * k[perm[s]];", "float bk = beta * k[s];"),
    "readout with k": ("column_sum_in(plain, f, perm, q, Tp.data(), ot.data());",
                       "column_sum_in(plain, f, perm, k, Tp.data(), ot.data());"),
    "f32 decay dropped": ("a[s] = (orc_row_kind(f, s) == ORC_KIND_INT) ? al * page->r[s] : al;",
                          "a[s] = (orc_row_kind(f, s) == ORC_KIND_INT) ? page->r[s] : 1.0f;"),
    "f64 decay dropped": ("AS[(size_t)kap * d_v + j] = al * Sij;", "AS[(size_t)kap * d_v + j] = Sij;"),
    "f64 prediction transposed": ("acc += (double)k[kap] * AS[(size_t)kap * d_v + j];",
                                  "acc += (double)k[j] * AS[(size_t)j * d_v + kap];"),
    "f64 beta dropped": ("+ (double)beta * (double)k[kap] * ((double)v[j] - pred[j]);",
                         "+ (double)k[kap] * ((double)v[j] - pred[j]);"),
    "row scale off by one": ("r = m / (float)qmax;", "r = m / (float)(qmax + 1);"),
    "rounding truncates": ("zr = std::nearbyint(x);", "zr = std::trunc(x);"),
    "bias wrong": ("int bias = (kind == ORC_KIND_INT) ? (1 << (bits - 1)) : 0;",
                   "int bias = (kind == ORC_KIND_INT) ? (1 << bits) - 1 : 0;"),
    "pcg4d xorshift dropped": ("    w ^= w >> 16;\n    x += y * w;", "    x += y * w;"),
    "pcg4d seed not mixed": ("b ^ (uint32_t)seed, h ^ (uint32_t)(seed >> 32) };", "b, h };"),
    "fp16 ties away": ("double n = std::nearbyint(t);\n    if (n >= 2048.0)",
                       "double n = std::floor(t + 0.5);\n    if (n >= 2048.0)"),
    "ranking ascending": ("return score[a] > score[b2];", "return score[a] < score[b2];"),
    "dequantize drops c": ("S_nat[(size_t)perm[s] * d_v + j] = (x * rs) * c;",
                           "S_nat[(size_t)perm[s] * d_v + j] = x * rs;"),
    "sr rounds up with 1 - frac": ("zr = (x >= fl + 1.0 - u) ? fl + 1.0 : fl;", "zr = (x >= fl + u) ? fl + 1.0 : fl;"),
    "sr offset on a 2^-17 grid": ("return (float)h16 * 0x1p-16f;", "return (float)h16 * 0x1p-17f;"),
    "sr halves swapped": ("uint32_t h16 = (j & 1) ? (word & 0xFFFFu) : (word >> 16);",
                          "uint32_t h16 = (j & 1) ? (word >> 16) : (word & 0xFFFFu);"),
    "column absmax over one row": ("float a = std::fabs(S_nat[(size_t)kap * d_v + j]);",
                                   "float a = std::fabs(S_nat[(size_t)j]);"),
    "window key decay dropped": ("K[(size_t)tau * d_k + kap] = K[(size_t)tau * d_k + kap] * al;",
                                 "K[(size_t)tau * d_k + kap] = K[(size_t)tau * d_k + kap];"),
    "window prediction with q": (
        "const float a = plain ? plain_dot(K + (size_t)tau * d_k, k, d_k) : lane_dot(K + (size_t)tau * d_k, k, d_k);",
        "const float a = plain ? plain_dot(K + (size_t)tau * d_k, q, d_k) : lane_dot(K + (size_t)tau * d_k, q, d_k);"),
    "window delta without beta": ("D[(size_t)t * d_v + j] = beta * e;", "D[(size_t)t * d_v + j] = e;"),
    "window readout skips this step": ("for (int tau = 0; tau <= t; ++tau) {\n        const float bq",
                                       "for (int tau = 0; tau < t; ++tau) {\n        const float bq"),
    "window commit drops the row factor": ("float x = Z[(size_t)s * d_v + j] * af[s];",
                                           "float x = Z[(size_t)s * d_v + j];"),
    "window row factor without decay": ("af[s] = P[kap] * rs;", "af[s] = rs;"),
    "window decay not reset": ("for (int kap = 0; kap < d_k; ++kap) P[kap] = 1.0f;",
                               "for (int kap = 0; kap < d_k; ++kap) P[kap] = P[kap];"),
    "window start keeps the old decay": ("const float p0 = (t == 0) ? 1.0f : P[kap];",
                                         "const float p0 = P[kap];"),
    "prefill later tokens not decayed": ("for (int j = 0; j < d_v; ++j) T[(size_t)s * d_v + j] = a_s * T[(size_t)s * d_v + j];",
                                         "for (int j = 0; j < d_v; ++j) T[(size_t)s * d_v + j] = T[(size_t)s * d_v + j];"),
    "prefill first beta for every token": ("const float bk = beta[l] * kl[perm[s]];", "const float bk = beta[0] * kl[perm[s]];"),
    "prefill readout with k": ("column_sum_in(plain, f, perm, ql, T.data(), ot.data());",
                               "column_sum_in(plain, f, perm, kl, T.data(), ot.data());"),
    "lifetime mean over samples only": ("const double mean = sum / ((double)n_samples * (double)B);",
                                        "const double mean = sum / (double)n_samples;"),
    "lifetime channel ignored": ("* H + h) * na + (f->gate_vector ? kap : 0)];", "* H + h) * na + 0];"),
    "lifetime head ignored": ("* H + h) * na + (f->gate_vector ? kap : 0)];",
                              "* H + 0) * na + (f->gate_vector ? kap : 0)];"),
    "lifetime first sample skipped": ("for (int t = 0; t < n_samples; ++t)\n                for (int b = 0; b < B; ++b)",
                                      "for (int t = 1; t < n_samples; ++t)\n                for (int b = 0; b < B; ++b)"),
    "plain chain skips channel 0": ("for (int kap = 0; kap < d_k; ++kap)\n            acc = std::fmaf(w_nat[kap], X[",
                                    "for (int kap = 1; kap < d_k; ++kap)\n            acc = std::fmaf(w_nat[kap], X["),
    "plain chain rows not permuted": ("for (int s = 0; s < d_k; ++s) row_of[perm[s]] = s;\n    for (int j = 0;",
                                      "for (int s = 0; s < d_k; ++s) row_of[s] = s;\n    for (int j = 0;"),
    "fit column rows not permuted": ("for (int s = 0; s < d_k; ++s) row_of[perm[s]] = s;\n    for (int it = 0;",
                                     "for (int s = 0; s < d_k; ++s) row_of[s] = s;\n    for (int it = 0;"),
    "plain dot skips the last channel": ("for (int i = 0; i < n; ++i) acc = std::fmaf(x[i], y[i], acc);",
                                         "for (int i = 0; i < n - 1; ++i) acc = std::fmaf(x[i], y[i], acc);"),
    "calibration skips request 0": ("for (int b = 0; b < B; ++b) {\n                const float *row",
                                    "for (int b = 1; b < B; ++b) {\n                const float *row"),
    "fit row scale ignores c": ("const double zc = (double)z[(size_t)s * d_v + j] * (double)c[j];",
                                "const double zc = (double)z[(size_t)s * d_v + j];"),
    "fit impact weights ignored": ("const double w = impact_nat ? (double)impact_nat[kap] : 1.0;",
                                   "const double w = 1.0;"),
    "fit codes truncate": ("double n = (d > 0.0) ? std::nearbyint((double)S_row[j] / d) : 0.0;",
                           "double n = (d > 0.0) ? std::trunc((double)S_row[j] / d) : 0.0;"),
    "chunk A without beta": ("                a *= bi;\n", "                a *= 1.0;\n"),
    "chunk decay from the wrong token": ("R(i, j, c) = R(i, j + 1, c) * gate(j + 1, c);",
                                         "R(i, j, c) = R(i, j + 1, c) * gate(j, c);"),
    "chunk A without the decay": ("a += (double)ki[c] * (double)kj[c] * R(i, jt, c);",
                                  "a += (double)ki[c] * (double)kj[c];"),
    "chunk readout skips the diagonal": ("for (int jt = 0; jt <= i; ++jt) {\n                const float *kj = k + (size_t)(t0 + jt) * d_k;\n                double pw",
                                         "for (int jt = 0; jt < i; ++jt) {\n                const float *kj = k + (size_t)(t0 + jt) * d_k;\n                double pw"),
    "chunk state keeps the old state undecayed": ("double acc = gn * S[(size_t)c * d_v + j];",
                                                  "double acc = S[(size_t)c * d_v + j];"),
    "window butterfly half": ("for (int off = lanes / 2; off >= 1; off /= 2) {",
                              "for (int off = lanes / 2; off >= 2; off /= 2) {"),
}


def _run_mutant(name, tmp):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, name
    d = os.path.join(tmp, "m%d" % list(MUTANTS).index(name))
    os.makedirs(d)
    shutil.copy(HDR, d)
    with open(os.path.join(d, "stq_oracle.cpp"), "w") as fh:
        fh.write(src.replace(old, new))
    lib = os.path.join(d, "libmut.so")
    subprocess.run(["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-o", lib,
                    os.path.join(d, "stq_oracle.cpp")], check=True)
    env = dict(os.environ, STQ_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider"] + PIN_FILES,
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            results = list(ex.map(lambda n: _run_mutant(n, tmp), MUTANTS))
    survivors = [n for n, rc in results if rc == 0]
    assert not survivors, "mutants not caught: %s" % survivors
