"""Build libsta.so (the product library), libsta_debug.so (the same sources
with the device-side bounds checks compiled in: -DSTA_DEBUG=1) and
libsta_probe.so (measurement probes) in-tree with nvcc for sm_100a.

    python block_sparse_attention_28_b200/build.py [--force]

Run it as a script (or load it by path): importing it through the package
would first load the library it is meant to (re)build.
"""
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "sta_lib.cu")
OUT = os.path.join(HERE, "libsta.so")
PROBE_SRC = os.path.join(HERE, "csrc", "sta_probe.cu")
PROBE_OUT = os.path.join(HERE, "libsta_probe.so")
DEBUG_OUT = os.path.join(HERE, "libsta_debug.so")
# (source, output, extra flags)
TARGETS = ((SRC, OUT, ()), (SRC, DEBUG_OUT, ("-DSTA_DEBUG=1",)), (PROBE_SRC, PROBE_OUT, ()))
NVCC_FLAGS = [
    "-O3", "-std=c++17",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-Xcompiler", "-fPIC",
    "-shared",
]


def _nvcc():
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libsta")
    return cand


def sources():
    d = os.path.join(HERE, "csrc")
    inc = os.path.join(os.path.dirname(HERE), "include")
    return [os.path.join(d, f) for f in sorted(os.listdir(d)) if f.endswith((".cu", ".cuh"))] + [
        os.path.join(inc, f) for f in sorted(os.listdir(inc)) if f.endswith(".h")]


def up_to_date(out=OUT):
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force=False, verbose=False):
    """Compile every target that is missing or older than a source; returns
    the path of libsta.so."""
    jobs = []
    for src, out, extra in TARGETS:
        if not force and up_to_date(out):
            continue
        cmd = [_nvcc(), *NVCC_FLAGS, *extra, "-o", out + ".tmp", src]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        jobs.append((subprocess.Popen(cmd), cmd, out))  # the targets compile side by side
    failed = None
    for proc, cmd, out in jobs:
        if proc.wait() != 0:
            failed = failed or subprocess.CalledProcessError(proc.returncode, cmd)
        else:
            os.replace(out + ".tmp", out)
    if failed is not None:
        raise failed
    return OUT


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(OUT)
