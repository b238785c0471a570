"""Build the C-ABI CUDA library ``libstq.so`` in-tree, for sm_100a only.

nvcc -gencode arch=compute_100a,code=sm_100a -O3 -lineinfo --fmad=false:
every fused multiply-add in the kernels is spelled out (__fmaf_rn,
__ffma2_rn), so the compiler contracts nothing and the fp32 evaluation order
is the one written in the source.
"""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libstq.so")
SOURCES = ["stq_api.cu", "stq_decode.cu", "stq_quant.cu", "stq_window.cu", "stq_prefill.cu", "stq_lifetime.cu", "stq_fit.cu", "stq_prefill_tc.cu"]
HEADERS = ["stq_device.cuh", "stq_internal.h", "stq_slices.cuh", "stq_rows.cuh", "stq_lifetime.h", "stq_tc.cuh"]

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "--fmad=false",
              "-std=c++17", "-Xcompiler", "-fPIC,-O2"]


def _inputs():
    return ([os.path.join(CSRC, s) for s in SOURCES + HEADERS]
            + [os.path.join(INCLUDE, "stq.h"), os.path.abspath(__file__)])


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every source to an object (in parallel: the files share no
    device code) and link the shared library; nothing is rebuilt while the
    library is newer than every input."""
    if not (force or stale()):
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB + ".tmp.%d" % os.getpid()
    with tempfile.TemporaryDirectory() as objdir:
        def compile_one(src):
            obj = os.path.join(objdir, os.path.splitext(src)[0] + ".o")
            cmd = [nvcc] + NVCC_FLAGS + (["-Xptxas", "-v"] if verbose else []) + \
                ["-I", INCLUDE, "-c", "-o", obj, os.path.join(CSRC, src)]
            subprocess.run(cmd, check=True)
            return obj
        with ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 1)) as ex:
            objs = list(ex.map(compile_one, SOURCES))
        subprocess.run([nvcc] + NVCC_FLAGS + ["-shared", "-o", tmp] + objs, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
