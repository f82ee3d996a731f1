"""Build step: compile the CUDA library in-tree for sm_100a.

``python -m paged_kv_cache_378_b200.build`` (or ``build()``) runs nvcc on
``csrc/pagedkv.cu`` and writes ``libpagedkv.so`` next to this file.  nvcc
cross-compiles, so this works on a machine without a GPU.  The library
carries a hash of its sources, header and flags (``pkv_build_hash``); the
loader rebuilds a library whose hash differs from the checkout's.
"""

import hashlib
import os
import re
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


BASE_FLAGS = ["-lineinfo", "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC"]
# the library carries the hash of what it was built from after this tag
HASH_TAG = b"PKV_BUILD_HASH:"


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


def source_hash(extra=()):
    """Hash of everything the library is built from: the CUDA sources, the
    C header and the compiler flags (16 hex digits)."""
    h = hashlib.sha256()
    for path in sources() + [os.path.join(INCLUDE, "pagedkv.h")]:
        h.update(os.path.basename(path).encode() + b"\0")
        with open(path, "rb") as f:
            h.update(f.read())
        h.update(b"\0")
    h.update(" ".join(ARCH_FLAGS + BASE_FLAGS + list(extra)).encode())
    return h.hexdigest()[:16]


def built_hash(path=LIB_PATH):
    """The source hash a built library carries, or None (no file, no tag)."""
    try:
        with open(path, "rb") as f:
            data = f.read()
    except OSError:
        return None
    m = re.search(re.escape(HASH_TAG) + rb"([0-9a-f]{16})", data)
    return m.group(1).decode() if m else None


def nvcc_path():
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: cannot build the pagedkv CUDA library")
    return cand


def build(verbose=False, out=LIB_PATH, extra=()):
    tag = f"-DPKV_BUILD_HASH=\"{source_hash(extra)}\""
    cmd = [nvcc_path(), *ARCH_FLAGS, *BASE_FLAGS, f"-I{INCLUDE}", tag, "-o", out,
           os.path.join(CSRC, "pagedkv.cu"), *extra]
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
    """True when the library is missing or was built from other sources."""
    return built_hash(path) != source_hash()


if __name__ == "__main__":
    build(verbose="-v" in sys.argv)
    print(LIB_PATH)
