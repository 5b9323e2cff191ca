"""Build libkvq.so (the CUDA library behind include/kvq.h) in-tree for sm_100a.

Each .cu file is compiled separately (in parallel) with nvcc for
-gencode arch=compute_100a,code=sm_100a, then linked into a shared library
next to this file.  No fast-math: the codec's decisions rely on IEEE sqrt and
division and on the documented accuracy of atan2f/log2f.

A library is reused only when the SHA-256 of every source, the public header,
this script and the compiler flags equals the digest recorded beside it
(libkvq.so.sha256) when it was built; anything else, including a library
copied in from elsewhere without its record, is rebuilt.
"""
from __future__ import annotations

import hashlib
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
OUT = os.path.join(HERE, "libkvq.so")
BUILD = os.path.join(ROOT, "_build")
SOURCES = ["kvq_abi.cu", "kvq_encode.cu", "kvq_dequant.cu", "kvq_decode.cu", "kvq_noalloc.cu",
           "kvq_decode_generic.cu", "kvq_debug.cu", "kvq_shard.cu"] + [
    f"kvq_decode_d{d}_g{g}.cu" for d in (64, 128) for g in (1, 2, 4, 8)]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


STAMP = OUT + ".sha256"


def source_digest(extra_flags=()) -> str:
    """SHA-256 over the names and contents of every input of the build and
    the flags it is compiled with."""
    files = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if not f.endswith(".py"))
    files += [os.path.join(ROOT, "include", "kvq.h"), os.path.abspath(__file__)]
    h = hashlib.sha256()
    for f in files:
        h.update(os.path.basename(f).encode() + b"\0")
        with open(f, "rb") as fh:
            h.update(fh.read())
    # the flags without the include directory's absolute path (it differs
    # between checkouts of the same sources)
    h.update(" ".join([f for f in (*FLAGS, *extra_flags) if not os.path.isabs(f)]).encode())
    return h.hexdigest()


def is_current(extra_flags=()) -> bool:
    """True when libkvq.so exists and was built from exactly these sources."""
    try:
        with open(STAMP) as f:
            return os.path.exists(OUT) and f.read().strip() == source_digest(extra_flags)
    except OSError:
        return False


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    if not force and is_current(extra_flags):
        return OUT
    digest = source_digest(extra_flags)
    os.makedirs(BUILD, exist_ok=True)

    def compile_one(src):
        obj = os.path.join(BUILD, src.replace(".cu", ".o"))
        cmd = [NVCC, *FLAGS, *extra_flags, "-c", os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout, r.stderr, file=sys.stderr)
        return obj

    with ThreadPoolExecutor(min(len(SOURCES), os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, SOURCES))
    tmp = OUT + f".tmp{os.getpid()}"
    # static CUDA runtime (nvcc's default): the library carries the runtime it
    # was compiled against instead of whichever libcudart the process has
    cmd = [NVCC, "-shared", "-cudart", "static", "-gencode", "arch=compute_100a,code=sm_100a",
           "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, OUT)
    with open(STAMP + f".tmp{os.getpid()}", "w") as f:
        f.write(digest + "\n")
    os.replace(STAMP + f".tmp{os.getpid()}", STAMP)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True,
                extra_flags=("-Xptxas", "-v") if "--ptxas-v" in sys.argv else ()))
