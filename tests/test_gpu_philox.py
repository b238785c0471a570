"""Pin of the oracle's Philox-4x32-10 in the counter word the host generator
cannot reach: cuRAND's device API (curand_init with a 64-bit subsequence,
then curand4) yields Philox(counter = (0, 0, sub mod 2^32, sub >> 32),
key = (seed mod 2^32, seed >> 32)).  A small program calling cuRAND is
compiled with nvcc at test time; its kernel writes one uint4 per thread.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle as O

pytestmark = pytest.mark.gpu

SRC = r"""
#include <cstdint>
#include <curand_kernel.h>
__global__ void draw(unsigned long long seed, const unsigned long long *subs, uint4 *out, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    curandStatePhilox4_32_10_t st;
    curand_init(seed, subs[i], 0, &st);
    out[i] = curand4(&st);
}
extern "C" int philox_draw(unsigned long long seed, const unsigned long long *h_subs, unsigned *h_out, int n) {
    unsigned long long *d_subs = nullptr;
    uint4 *d_out = nullptr;
    if (cudaMalloc(&d_subs, n * sizeof(unsigned long long)) != cudaSuccess) return 1;
    if (cudaMalloc(&d_out, n * sizeof(uint4)) != cudaSuccess) return 2;
    cudaMemcpy(d_subs, h_subs, n * sizeof(unsigned long long), cudaMemcpyHostToDevice);
    draw<<<(n + 127) / 128, 128>>>(seed, d_subs, d_out, n);
    cudaError_t err = cudaMemcpy(h_out, d_out, n * sizeof(uint4), cudaMemcpyDeviceToHost);
    cudaFree(d_subs);
    cudaFree(d_out);
    return err == cudaSuccess ? 0 : 3;
}
"""


@pytest.fixture(scope="module")
def draw(tmp_path_factory):
    d = tmp_path_factory.mktemp("philox")
    src, lib = d / "draw.cu", d / "libdraw.so"
    src.write_text(SRC)
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared", "-Xcompiler", "-fPIC",
                    "-o", str(lib), str(src)], check=True)
    L = ctypes.CDLL(str(lib))
    L.philox_draw.restype = ctypes.c_int
    L.philox_draw.argtypes = [ctypes.c_ulonglong, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]

    def run(seed, subs):
        subs = np.ascontiguousarray(subs, np.uint64)
        out = np.zeros((len(subs), 4), np.uint32)
        assert L.philox_draw(seed, subs.ctypes.data, out.ctypes.data, len(subs)) == 0
        return out
    return run


def test_philox_fourth_counter_word_matches_curand_device(draw):
    rng = np.random.default_rng(77)
    for seed in (0, 2**64 - 1, int(rng.integers(0, 2**63))):
        subs = [int(rng.integers(0, 2**64, dtype=np.uint64)) for _ in range(61)] + [2**32, 2**64 - 1, 5 << 32]
        got = draw(seed, subs)
        key = np.array([seed & 0xFFFFFFFF, seed >> 32], np.uint32)
        for sub, row in zip(subs, got):
            ctr = np.array([0, 0, sub & 0xFFFFFFFF, sub >> 32], np.uint32)
            assert np.array_equal(O.philox4x32_10(ctr, key), row), (seed, sub)
