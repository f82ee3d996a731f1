"""Build step: compile the CUDA library in-tree for sm_100a.

``python -m paged_kv_cache_378_b200.build`` (or ``build()``) runs nvcc on
``csrc/pagedkv.cu`` and writes ``libpagedkv.so`` next to this file.  nvcc
cross-compiles, so this works on a machine without a GPU.
"""

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libpagedkv.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


def nvcc_path():
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: cannot build the pagedkv CUDA library")
    return cand


def build(verbose=False, out=LIB_PATH, extra=()):
    cmd = [nvcc_path(), *ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", f"-I{INCLUDE}", "-o", out, os.path.join(CSRC, "pagedkv.cu"), *extra]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    tmp = f"{out}.{os.getpid()}.tmp"
    cmd[cmd.index(out)] = tmp
    res = subprocess.run(cmd, capture_output=not verbose, text=True)
    if res.returncode != 0:
        msg = (res.stderr or "") + (res.stdout or "")
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{msg}")
    os.replace(tmp, out)
    return out


def needs_build(path=LIB_PATH):
    return not os.path.exists(path)


if __name__ == "__main__":
    build(verbose="-v" in sys.argv)
    print(LIB_PATH)
