"""Build libpa.so in-tree with nvcc for sm_100a.

``python -m paged_kv_cache_418_b200._build`` (or ``ensure_built()``) compiles
every ``csrc/*.cu`` into ``paged_kv_cache_418_b200/libpa.so`` and records a
hash of the sources and flags beside it, so a stale library is rebuilt.
"""

from __future__ import annotations

import glob
import hashlib
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libpa.so")
STAMP = LIB + ".src-sha256"

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
              "-Xptxas", "-warn-spills"] + ARCH


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _hash() -> str:
    h = hashlib.sha256()
    files = _sources() + sorted(glob.glob(os.path.join(CSRC, "*.h")) +
                                glob.glob(os.path.join(CSRC, "*.cuh")))
    files.append(os.path.join(ROOT, "include", "pa.h"))
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    h.update(" ".join(NVCC_FLAGS).encode())
    return h.hexdigest()


def is_current() -> bool:
    if not (os.path.exists(LIB) and os.path.exists(STAMP)):
        return False
    with open(STAMP) as f:
        return f.read().strip() == _hash()


def build(verbose: bool = False) -> str:
    """Compile all CUDA sources (in parallel) and link libpa.so."""
    nvcc = _nvcc()
    h = _hash()
    with tempfile.TemporaryDirectory(prefix="pa_build_") as tmp:
        objs = []

        def compile_one(src):
            obj = os.path.join(tmp, os.path.basename(src) + ".o")
            cmd = [nvcc, *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stderr}")
            if verbose and r.stderr.strip():
                sys.stderr.write(r.stderr)
            return obj

        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            objs = list(ex.map(compile_one, _sources()))
        tmp_lib = os.path.join(tmp, "libpa.so")
        cmd = [nvcc, *ARCH, "-shared", "-o", tmp_lib, *objs, "-cudart", "static"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc link failed:\n{r.stderr}")
        shutil.copyfile(tmp_lib, LIB + ".tmp")
        os.replace(LIB + ".tmp", LIB)
    with open(STAMP, "w") as f:
        f.write(h)
    return LIB


def ensure_built() -> str:
    if not is_current():
        build()
    return LIB


if __name__ == "__main__":
    print(build(verbose=True))
