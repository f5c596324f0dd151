"""Build libkvq.so (CUDA, sm_100a) into kv_cache_bit_b200/_lib/.

nvcc cross-compiles without a GPU.  The library is a single translation unit
(csrc/kvq_api.cu, which includes the kernel headers).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT_DIR = os.path.join(HERE, "_lib")
LIB = os.path.join(OUT_DIR, "libkvq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


TEST_LIB = os.path.join(OUT_DIR, "libkvq_waittest.so")


def _cmd(out, extra=()):
    return [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
            "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
            "--expt-relaxed-constexpr", *extra, "-o", out + ".tmp", os.path.join(CSRC, "kvq_api.cu")]


def build(force: bool = False, verbose: bool = False, test_lib: bool = True) -> str:
    """Build libkvq.so and, unless test_lib is False, the test build
    libkvq_waittest.so (the same sources with KVQ_WAIT_TEST: the kernels'
    main-loop waits can be made to give up at once, for the failure-path
    test).  The two compile in parallel."""
    os.makedirs(OUT_DIR, exist_ok=True)
    deps = sources() + [os.path.join(ROOT, "include", "kvq.h"), __file__]
    newest = max(os.path.getmtime(p) for p in deps)
    jobs = []
    targets = [(LIB, ())] + ([(TEST_LIB, ("-DKVQ_WAIT_TEST",))] if test_lib else [])
    for out, extra in targets:
        if force or not os.path.exists(out) or os.path.getmtime(out) < newest:
            cmd = _cmd(out, extra)
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
            jobs.append((out, subprocess.Popen(cmd)))
    for out, proc in jobs:
        if proc.wait() != 0:
            raise subprocess.CalledProcessError(proc.returncode, "nvcc " + out)
        os.replace(out + ".tmp", out)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
