"""Build the sm_100a C-ABI library ``libmsa_b200.so`` in-tree with nvcc.

Every kernel source in ``csrc/`` is compiled for ``sm_100a`` only and linked
into one shared library that exports the functions declared in
``include/msa.h``.  Objects are cached under ``_build/`` by source hash.
"""
from __future__ import annotations

import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libmsa_b200.so")
HEADER = os.path.join(ROOT, "include", "msa.h")

SOURCES = ["api.cu", "index_kernel.cu", "csr_kernel.cu", "main_kernel.cu", "merge_kernel.cu",
           "align_kernel.cu", "quant_kernel.cu", "mx_kernel.cu",
           "decode_kernel.cu", "decode_static.cu", "selftest.cu"]
NVCC = os.environ.get("NVCC", "nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
         "-Xptxas", "-warn-spills", f"-I{CSRC}", f"-I{os.path.join(ROOT, 'include')}"]


def _deps_hash() -> str:
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + f.read())
    with open(HEADER, "rb") as f:
        h.update(f.read())
    # the flags without the include paths: those are absolute and differ between
    # checkouts of the same sources
    h.update(" ".join(f for f in FLAGS if not f.startswith("-I")).encode())
    return h.hexdigest()[:16]


def is_current() -> bool:
    """True when the library exists and was built from the current sources."""
    stamp = os.path.join(BUILD, "stamp")
    if not (os.path.exists(LIB) and os.path.exists(stamp)):
        return False
    with open(stamp) as f:
        return f.read().strip() == _deps_hash()


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    tag = _deps_hash()
    stamp = os.path.join(BUILD, "stamp")
    if not force and os.path.exists(LIB) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == tag:
                return LIB
    objs = []
    for src in SOURCES:
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        cmd = [NVCC, *FLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp,
                    *objs, "-lcudart"], check=True)
    os.replace(tmp, LIB)
    with open(stamp, "w") as f:
        f.write(tag)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
