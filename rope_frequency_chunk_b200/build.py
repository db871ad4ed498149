"""Builds libfasa.so in-tree for sm_100a with nvcc (no JIT cache, no install).

    python -m rope_frequency_chunk_b200.build [--verbose]
"""
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfasa.so")
SOURCES = ["fasa.cu"]
DEPS = ["fasa.cu", "fasa_device.cuh", "append.cuh", "score.cuh", "select_attend.cuh", "select_hist.cuh", "decode_wide.cuh", "tip.cuh", "attend_cc.cuh", "attend_mma.cuh", "attend_tc.cuh", "calibrate.cuh"]
HEADER = os.path.join(os.path.dirname(HERE), "include", "fasa.h")


def nvcc() -> str:
    for c in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def flags(ptxas_verbose=False):
    f = ["-std=c++17", "-O3", "-lineinfo", "-gencode", "arch=compute_100a,code=sm_100a",
         "-Xcompiler", "-fPIC", "-shared", "-diag-suppress", "177"]
    if ptxas_verbose:
        f += ["-Xptxas", "-v"]
    return f


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    srcs = [os.path.join(CSRC, d) for d in DEPS] + [HEADER]
    return all(os.path.getmtime(s) <= t for s in srcs)


def build(force=False, verbose=False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [nvcc()] + flags(verbose) + ["-o", LIB + ".tmp"] + [os.path.join(CSRC, s) for s in SOURCES]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="--verbose" in sys.argv))
