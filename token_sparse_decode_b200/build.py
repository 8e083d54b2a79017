"""Build the C-ABI library libaoh.so for sm_100a (in-tree, next to this file).

    python -m token_sparse_decode_b200.build [--ptxas-verbose]

The library is one translation unit (csrc/aoh_api.cu includes the kernels) linked
against the shared CUDA runtime, so that it shares the runtime instance (current
device, streams) of the PyTorch process that loads it.  A rebuild happens whenever
the sha256 of the sources and flags differs from the one recorded beside the
library (libaoh.so.srchash), whatever the files' times.
"""

from __future__ import annotations

import hashlib
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "aoh_api.cu")
OUT = os.path.join(HERE, "libaoh.so")
HASH = OUT + ".srchash"  # source hash the library was built from
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    d = os.path.join(HERE, "csrc")
    return sorted(os.path.join(d, f) for f in os.listdir(d)) + [os.path.join(ROOT, "include", "aoh.h")]


def _command(out: str) -> list:
    return [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
            "-cudart", "shared", "-I", os.path.join(ROOT, "include"), "-I", os.path.join(HERE, "csrc"),
            "-o", out, SRC]


def source_hash() -> str:
    """sha256 of every source file (name and bytes) and of the compile flags."""
    h = hashlib.sha256()
    for path in _sources():
        h.update(os.path.basename(path).encode() + b"\0")
        with open(path, "rb") as f:
            h.update(f.read())
    h.update(" ".join(_command("libaoh.so")[1:]).encode())
    return h.hexdigest()


def up_to_date() -> bool:
    """The library exists and was built from exactly the current sources and flags."""
    if not (os.path.exists(OUT) and os.path.exists(HASH)):
        return False
    with open(HASH) as f:
        return f.read().strip() == source_hash()


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and up_to_date():
        return OUT
    digest = source_hash()
    cmd = _command(OUT + ".tmp")
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if ptxas_verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(OUT + ".tmp", OUT)
    with open(HASH, "w") as f:
        f.write(digest + "\n")
    return OUT


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--ptxas-verbose" in sys.argv))
