"""Build libesa.so in-tree for sm_100a with nvcc (one translation unit)."""
from __future__ import annotations

import hashlib
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "esa_lib.cu")
OUT = os.path.join(HERE, "libesa.so")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17", "-shared",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-O2"]


def nvcc_path() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def sources():
    d = os.path.join(HERE, "csrc")
    return [os.path.join(d, f) for f in sorted(os.listdir(d)) if f.endswith((".cu", ".cuh"))] + \
        [os.path.join(os.path.dirname(HERE), "include", "esa.h")]


STAMP = OUT + ".sha256"


def source_hash(extra_flags=()) -> str:
    """SHA-256 over every source the library is built from (names and contents) and
    the compiler flags: the binary is reused only when this matches the hash recorded
    beside it at its build, whatever the files' modification times."""
    h = hashlib.sha256()
    for f in sources():
        h.update(os.path.basename(f).encode() + b"\0")
        with open(f, "rb") as fh:
            h.update(fh.read())
        h.update(b"\0")
    h.update(" ".join([*NVCC_FLAGS, *extra_flags]).encode())
    return h.hexdigest()


def up_to_date(extra_flags=()) -> bool:
    if not (os.path.exists(OUT) and os.path.exists(STAMP)):
        return False
    with open(STAMP) as fh:
        return fh.read().strip() == source_hash(extra_flags)


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    """Compile csrc/esa_lib.cu into libesa.so next to this file. Returns its path."""
    if not force and up_to_date(extra_flags):
        return OUT
    digest = source_hash(extra_flags)
    cmd = [nvcc_path(), *NVCC_FLAGS, *extra_flags, "-o", OUT + ".tmp", SRC]
    if verbose:
        print(" ".join(cmd))
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libesa")
    os.replace(OUT + ".tmp", OUT)
    with open(STAMP, "w") as fh:
        fh.write(digest + "\n")
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
