"""Build step for libsmla.so (the C-ABI library with the sm_100a kernels).

Compiles every ``csrc/*.cu`` with nvcc for sm_100a into
``sparse_mla_decoding_b200/libsmla.so`` (in-tree, so it travels with the
repository snapshot), then applies the register-spill gate: the build fails if
ptxas reports any spill stores or loads, unless SMLA_SKIP_REG_SPILL_CHECK=1.
A sidecar file records a hash of the sources so stale builds are detected.
"""
from __future__ import annotations

import glob
import hashlib
import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libsmla.so")
STAMP = LIB + ".srchash"
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def source_hash() -> str:
    h = hashlib.sha256()
    files = sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")))
    files += [os.path.join(INCLUDE, "smla.h"), os.path.abspath(__file__)]
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def is_current() -> bool:
    if not os.path.exists(LIB) or not os.path.exists(STAMP):
        return False
    with open(STAMP) as f:
        return f.read().strip() == source_hash()


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and is_current():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-Xptxas", "-v",
           "-I", INCLUDE, "-o", tmp, *sources()]
    res = subprocess.run(cmd, capture_output=True, text=True)
    log = res.stdout + res.stderr
    if res.returncode != 0:
        sys.stderr.write(log)
        raise RuntimeError("nvcc failed building libsmla.so")
    spills = [(int(a), int(b)) for a, b in re.findall(r"(\d+) bytes spill stores, (\d+) bytes spill loads", log)]
    if any(a or b for a, b in spills) and os.environ.get("SMLA_SKIP_REG_SPILL_CHECK") != "1":
        sys.stderr.write(log)
        os.remove(tmp)
        raise RuntimeError("register spilling detected in libsmla.so (set SMLA_SKIP_REG_SPILL_CHECK=1 to skip)")
    if verbose:
        sys.stdout.write(log)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(source_hash())
    with open(LIB + ".ptxas.log", "w") as f:
        f.write(log)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
