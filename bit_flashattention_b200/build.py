"""Build the CUDA libraries in-tree for sm_100a with nvcc.

libhifa4.so       the product library: the C ABI of include/hifa4.h.
libhifa4_test.so  the same sources built with HIFA4_TEST_HOOKS: the product ABI plus the
                  test-only exports of include/hifa4_test.h (tile probes, fault
                  injection).  Only the tests load it.
libhifa4_peak.so  the dense FP4 tensor-core rate loop of include/hifa4_peak.h, which
                  bench.py uses as the attention's roofline peak.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRCS = [os.path.join(HERE, "csrc", f) for f in ("hifa4_api.cu", "hifa4_noalloc.cu", "calib_file.cpp")]
# every header the translation units include: a change to any of them rebuilds
DEPS = sorted(os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc")) if f.endswith(".cuh")) + \
       [os.path.join(ROOT, "include", "hifa4.h"), os.path.join(ROOT, "include", "hifa4_test.h")]
LIB = os.path.join(HERE, "libhifa4.so")
TEST_LIB = os.path.join(HERE, "libhifa4_test.so")
PEAK_LIB = os.path.join(HERE, "libhifa4_peak.so")
PEAK_SRCS = [os.path.join(HERE, "csrc", "fp4_peak.cu")]
PEAK_DEPS = [os.path.join(HERE, "csrc", "ptx.cuh"), os.path.join(ROOT, "include", "hifa4_peak.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--fmad=false",                 # no implicit multiply-add contraction: results follow the written rounding steps
    "-Xcompiler", "-fPIC", "-shared",
    "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def _stale(lib: str, inputs) -> bool:
    newest = max(os.path.getmtime(p) for p in list(inputs) + [os.path.abspath(__file__)])
    return not os.path.exists(lib) or os.path.getmtime(lib) < newest


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile whichever of the libraries is out of date (all at once, in parallel)."""
    jobs = []
    for lib, extra, srcs, deps in ((LIB, [], SRCS, DEPS), (TEST_LIB, ["-DHIFA4_TEST_HOOKS"], SRCS, DEPS),
                                   (PEAK_LIB, [], PEAK_SRCS, PEAK_DEPS)):
        if force or _stale(lib, srcs + deps):
            cmd = [nvcc()] + NVCC_FLAGS + extra + (["-Xptxas", "-v"] if verbose else []) + ["-o", lib] + srcs
            jobs.append((cmd, subprocess.Popen(cmd)))
    for cmd, p in jobs:
        if p.wait() != 0:
            raise subprocess.CalledProcessError(p.returncode, cmd)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
    print(LIB)
    print(TEST_LIB)
    print(PEAK_LIB)
